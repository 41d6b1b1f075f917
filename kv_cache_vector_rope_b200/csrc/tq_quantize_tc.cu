// Tensor-core quantiser (sm_100a, tcgen05) for bf16 inputs, d in {64, 128},
// one shared Pi, no RoPE (the post-RoPE K/V of the ESM- and Llama-shaped
// caches). Computes exactly what tq_quantize_kv specifies; codes and signs are
// those of exact arithmetic (see "Exactness").
//
// Sources: 7minutos.es "KV cache ... TurboQuant" Etapa 1 (y = Pi x, Lloyd-Max
// index per coordinate of y/||x||) and Etapa 2 (sign of S times the residual,
// residual norm); gist.science "TurboESM ..." section 2A (RoPE before Pi).
//
// Per CTA (persistent, one per SM), tiles of 128 vectors; tile i of a CTA
// uses TMEM slot i % 2 and is finished by epilogue warpgroup i % 2, so the two
// warpgroups work on alternate tiles and never wait for each other:
//   warp 0      TMA: 128 x d bf16 tile -> shared memory (128-byte swizzle),
//               2-4 stage ring; a stage is released by the MMA that read it
//   warp 1      TMEM owner and single-thread MMA issuer:
//                 Y = X (Pi3 + Pi2 + Pi1)^T      bf16 splits, small parts first
//                 P = (R1 + R2) (S1 + S2)^T      fp16 splits, A from TMEM
//                                                (R2 S1 + R1 S2 + R1 S1)
//   warps 2-5   epilogue warpgroup 0, warps 6-9 epilogue warpgroup 1; thread =
//               vector (TMEM lane). Per tile, in 32-column chunks (a loop that is
//               not unrolled across chunks, so the epilogue stays in the
//               instruction cache): ||y|| from the accumulator; codes by binary
//               search against ||y|| t_j (by |y| against t_4..t_6 when the
//               3-bit table is exactly symmetric); residual r and the fp16
//               splits of r 2^k (k from ||y||, so r 2^k stays below 2^14) into
//               TMEM for P; sign bits from P; packing and stores per chunk.
// TMEM slot (keys): Y/P accumulator (d columns) | R1 (d/2) | R2 (d/2).
//
// Exactness. The norm is ||y|| = ||Pi x|| in fp32 (Pi orthogonal; error
// ~1e-7 relative). A code is decided in fp32 only when y is farther than
// 3e-7 ||y|| from every boundary it was compared with, a sign only when |p|
// exceeds 1.5e-5 ||r||. A row with any other coordinate or sign is flagged
// (sign bit of its stored ||r|| for keys, of ||x|| for values) and a second
// launch, quantize_fixup, recomputes every flagged row exactly in fp64 (four
// rows per warp: ||x||, y = Pi x, codes, r, p = S r) and overwrites it.
//
// Every wait is bounded (2 s; the pipeline waits take the launch's limit, which
// the environment variable TQ_TEST_WAIT_NS can shorten); a timeout sets
// TQ_DEV_TIMEOUT in *d_status and the CTA drains its own copies and MMAs (full
// 2 s limit), frees TMEM and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <mutex>
#include <type_traits>

#include "tq_device.cuh"
#include "tq_internal.h"
#include "tq_sm100.cuh"
#include "tq_tc.h"

namespace tq {
namespace {

using namespace sm100;
using dev::warp_sum;

constexpr int kThreads = 320;         // 10 warps
// Guard bands, set from the measured errors of this formulation on B200: the
// rotation accumulator errs by at most 7.4e-8 ||x|| per coordinate (typically
// 2e-8), and the projection of the fp32 residual by at most 2.5e-6 ||r||
// (the residual inherits the rotation's error). Each band is 4-6x the
// largest error seen over ~5e5 samples.
constexpr float kCodeGuard = 3e-7f;
constexpr float kSignGuard = 1.5e-5f;

constexpr int pow2_at_least(int x) {
  int p = 32;
  while (p < x) p <<= 1;
  return p;
}

template <int D, bool KEY, bool PH = false>
struct Cfg {
  static constexpr int kM = 128;
  static constexpr int kKSteps = D / 16;
  static constexpr int kTileBytes = kM * D * 2;
  static constexpr int kMatBytes = D * D * 2;
  static constexpr int kStages = (D == 128) ? (KEY ? 2 : 3) : 4;
  static constexpr int kSSplits = KEY ? 2 : 0;
  static constexpr int kSlotCols = KEY ? 2 * D : D;  // accumulator | R1 | R2
  static constexpr int kColR1 = D;
  static constexpr int kColR2 = D + D / 2;
  static constexpr int kTmemCols = pow2_at_least(2 * kSlotCols);
  static constexpr int kChunks = D / 32;             // 32-column chunks
  // Shared memory plan (offsets from a 1024-aligned base).
  // Pi splits: one slot, or two (per-head mode: the next head's Pi is
  // written into the other slot while the current one is in use).
  static constexpr int kPiSlot = 3 * kMatBytes;
  static constexpr int kOffPi = 0;
  static constexpr int kOffS = kOffPi + (PH ? 2 : 1) * kPiSlot;
  static constexpr int kOffX = kOffS + kSSplits * kMatBytes;
  static constexpr int kOffBar = kOffX + kStages * kTileBytes;
  // full[st], empty[st], yfull[2], rfull[2], pfull[2], accfree[2], drain,
  // pi_full[2], pi_free[2]
  static constexpr int kNumBars = 2 * kStages + 8 + 1 + 4;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  // misc: tmem base (4) + abort (4) + r-scale exponent shift (4) + symmetric-table flag (4) + cent[16] + bnd[16]
  static constexpr int kOffCent = kOffMisc + 16;
  static constexpr int kOffBnd = kOffCent + 64;
  static constexpr int kSmemBytes = kOffBnd + 64 + 1024;   // + alignment slack
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
  uint64_t wait_ns;     // pipeline wait limit (drains keep 2 s)
  int64_t vpp;          // vectors per rotation (per-head mode)
  int64_t pi_stride;    // floats between rotations; 0: one shared Pi
};

// Splits v into bf16 terms hi + mid + lo that add up to v to ~2^-25.
__device__ __forceinline__ void split3(float v, __nv_bfloat16& a, __nv_bfloat16& b, __nv_bfloat16& c) {
  a = __float2bfloat16_rn(v);
  const float r1 = v - __bfloat162float(a);
  b = __float2bfloat16_rn(r1);
  c = __float2bfloat16_rn(r1 - __bfloat162float(b));
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

// Code of y against thresholds th[] (strict: ties go to the lower code);
// `near` is set when y lies within `band` of a boundary it was compared with
// (the boundaries of its cell are among them).
template <int BITS>
__device__ __forceinline__ int code_guarded(float y, const float (&th)[(1 << BITS) - 1], float band, bool& near) {
  if constexpr (BITS == 3) {
    const bool b2 = y > th[3];
    const float tA = b2 ? th[5] : th[1];
    const bool b1 = y > tA;
    const float tB = b2 ? (b1 ? th[6] : th[4]) : (b1 ? th[2] : th[0]);
    const bool b0 = y > tB;
    near |= (fabsf(y - th[3]) < band) | (fabsf(y - tA) < band) | (fabsf(y - tB) < band);
    return (b2 ? 4 : 0) | (b1 ? 2 : 0) | (b0 ? 1 : 0);
  } else if constexpr (BITS == 2) {
    const bool b1 = y > th[1];
    const float tA = b1 ? th[2] : th[0];
    const bool b0 = y > tA;
    near |= (fabsf(y - th[1]) < band) | (fabsf(y - tA) < band);
    return (b1 ? 2 : 0) | (b0 ? 1 : 0);
  } else {
    int c = 0;
#pragma unroll
    for (int j = 0; j < (1 << BITS) - 1; ++j) {
      c += (y > th[j]) ? 1 : 0;
      near |= fabsf(y - th[j]) < band;
    }
    return c;
  }
}

// 3-bit code for a symmetric table (t_{6-j} = -t_j, t_3 = 0): the sign of y
// picks the half, |y| is searched against t_4 < t_5 < t_6, and the code is
// 4 + m (y > 0) or 3 - m. A tie |y| = t_j, where the two rules could differ,
// lies inside the guard band and flags the row like every other near value.
template <int NB>
__device__ __forceinline__ int code_symmetric3(float y, const float (&th)[NB], float band, bool& near) {
  const float ay = fabsf(y);
  const bool b1 = ay > th[5];
  const float tB = b1 ? th[6] : th[4];
  const bool b0 = ay > tB;
  near |= (ay < band) | (fabsf(ay - th[5]) < band) | (fabsf(ay - tB) < band);
  const int m = (b1 ? 2 : 0) | (b0 ? 1 : 0);
  return (y > 0.f ? 4 : 3) ^ m;
}

// bf16 splits hi + mid + lo of Pi into one slot (three K-major, 128B-swizzled
// matrices), elements first, first + step, ...
template <int D>
__device__ __forceinline__ void stage_pi3(unsigned char* slot, const float* __restrict__ Pi, int first, int step) {
  constexpr int kMat = D * D * 2;
#pragma unroll 4
  for (int e = first; e < D * D; e += step) {
    const uint32_t off = sw128_offset(e / D, e % D, D);
    __nv_bfloat16 h, m, l;
    split3(__ldg(Pi + e), h, m, l);
    *reinterpret_cast<__nv_bfloat16*>(slot + off) = h;
    *reinterpret_cast<__nv_bfloat16*>(slot + kMat + off) = m;
    *reinterpret_cast<__nv_bfloat16*>(slot + 2 * kMat + off) = l;
  }
}

// PH (per-head mode, d = 64): vector v uses Pi + (v / vpp) pi_stride, with vpp
// a multiple of the 128-vector tile. Each CTA then takes a contiguous range of
// tiles, and the producer warp writes each new head's Pi splits into the slot
// the head before last used (pi_free), announcing them with pi_full.
template <int D, bool KEY, int BITS, bool PH>
__global__ void __launch_bounds__(kThreads, 1) quantize_tc_kernel(const __grid_constant__ CUtensorMap tmap, TcArgs a) {
  using C = Cfg<D, KEY, PH>;
  constexpr int kNb = (1 << BITS) - 1;
  constexpr int kRowBytes = D * BITS / 8;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* pi_s = sm + C::kOffPi;
  unsigned char* s_s = sm + C::kOffS;
  unsigned char* x_s = sm + C::kOffX;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + C::kOffBar);
  uint64_t* full = bars;
  uint64_t* empty = bars + C::kStages;
  uint64_t* yfull = bars + 2 * C::kStages;           // [2]
  uint64_t* rfull = yfull + 2;                        // [2]
  uint64_t* pfull = rfull + 2;                        // [2]
  uint64_t* accfree = pfull + 2;                      // [2]
  uint64_t* drain = accfree + 2;                      // [1] final MMA drain
  uint64_t* pi_full = drain + 1;                      // [2] per-head mode: Pi slot written
  uint64_t* pi_free = pi_full + 2;                    // [2] per-head mode: MMAs done with the slot
  uint32_t* tmem_base_s = reinterpret_cast<uint32_t*>(sm + C::kOffMisc);
  volatile int* abort_s = reinterpret_cast<volatile int*>(sm + C::kOffMisc + 4);
  int* rshift_s = reinterpret_cast<int*>(sm + C::kOffMisc + 8);
  int* sym_s = reinterpret_cast<int*>(sm + C::kOffMisc + 12);
  float* cent_s = reinterpret_cast<float*>(sm + C::kOffCent);
  float* bnd_s = reinterpret_cast<float*>(sm + C::kOffBnd);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t n_tiles = (a.n + C::kM - 1) / C::kM;
  // Tiles of this CTA: every gridDim.x-th (shared Pi), or a contiguous range
  // (per-head mode: few head changes per CTA).
  const int64_t ph_lo = n_tiles * blockIdx.x / gridDim.x, ph_hi = n_tiles * (blockIdx.x + 1) / gridDim.x;
  const int my_tiles = PH ? static_cast<int>(ph_hi - ph_lo)
                          : (n_tiles > blockIdx.x) ? static_cast<int>((n_tiles - blockIdx.x + gridDim.x - 1) / gridDim.x)
                                                   : 0;
  auto tile_of = [&](int it) -> int64_t { return PH ? ph_lo + it : blockIdx.x + int64_t(it) * gridDim.x; };
  auto head_of = [&](int64_t t) -> int64_t { return PH ? t * C::kM / a.vpp : 0; };

  // ---------------------------------------------------------------- prologue
  if (tid == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&yfull[b], 1);
      mbar_init(&rfull[b], 4);
      mbar_init(&pfull[b], 1);
      mbar_init(&accfree[b], 4);
    }
    mbar_init(drain, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&pi_full[b], 1);
      mbar_init(&pi_free[b], 1);
    }
    *abort_s = 0;
    // r 2^k must stay below 2^14 for fp16: |r| <= (1 + max|c|) ||y||.
    float lim = 1.f;
    for (int k = 0; k <= kNb; ++k) lim = fmaxf(lim, 1.f + fabsf(a.cent[k]));
    int sh = 0;
    while (lim > 2.f && sh < 60) {
      lim *= 0.5f;
      ++sh;
    }
    *rshift_s = sh;
    // Exactly symmetric 3-bit boundaries (the analytic tables are).
    bool sy = BITS == 3 && a.bnd[3] == 0.f;
    for (int j = 0; j < kNb; ++j) sy = sy && (a.bnd[j] == -a.bnd[kNb - 1 - j]);
    *sym_s = sy ? 1 : 0;
    mbar_fence_init();
  }
  if (tid < 16) cent_s[tid] = tid <= kNb ? a.cent[tid] : 0.f;
  if (tid < 16) bnd_s[tid] = tid < kNb ? a.bnd[tid] : 0.f;
  if (warp == 1) {
    tmem_alloc(tmem_base_s, C::kTmemCols);
    tmem_relinquish();
  }
  // bf16 splits of Pi (3) and fp16 splits of S (2), K-major, 128B-swizzled
  // (per-head mode: the producer stages each head's Pi).
  if (!PH) stage_pi3<D>(pi_s, a.Pi, tid, kThreads);
  for (int e = tid; e < D * D; e += kThreads) {
    const int i = e / D, j = e % D;
    const uint32_t off = sw128_offset(i, j, D);
    if (KEY) {
      const float sv = __ldg(a.S + e);
      const __half sh = __float2half_rn(sv);
      const __half sl = __float2half_rn(sv - __half2float(sh));
      *reinterpret_cast<__half*>(s_s + off) = sh;
      *reinterpret_cast<__half*>(s_s + C::kMatBytes + off) = sl;
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
    // The whole warp runs the loop (it stages the per-head Pi splits); lane 0
    // issues the tile loads.
    int armed[C::kStages];
    for (int s = 0; s < C::kStages; ++s) armed[s] = 0;
    int64_t cur_head = -1;
    int nh = 0;                                   // heads staged so far
    for (int it = 0; it < my_tiles; ++it) {
      const int64_t t = tile_of(it);
      if (PH) {
        const int64_t h = head_of(t);
        if (h != cur_head) {
          const int slot = nh & 1;
          bool ok = *abort_s == 0;
          if (ok && nh >= 2) ok = mbar_wait(&pi_free[slot], ((nh - 2) >> 1) & 1, a.wait_ns);
          if (!__all_sync(0xffffffffu, ok)) {
            if (lane == 0 && !*abort_s) fail();
            break;
          }
          stage_pi3<D>(pi_s + slot * C::kPiSlot, a.Pi + h * a.pi_stride, lane, 32);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&pi_full[slot]);
          cur_head = h;
          ++nh;
        }
      }
      int go = 1;
      if (lane == 0) {
        const int st = it % C::kStages;
        const uint32_t ph = (it / C::kStages) & 1;
        if (*abort_s) {
          go = 0;
        } else if (!mbar_wait(&empty[st], ph ^ 1, a.wait_ns)) {
          fail();
          go = 0;
        } else {
          mbar_expect_tx(&full[st], C::kTileBytes);
          unsigned char* dst = x_s + st * C::kTileBytes;
#pragma unroll
          for (int k = 0; k < D / 64; ++k) tma_load_2d(dst + k * C::kM * 128, &tmap, &full[st], k * 64, int(t * C::kM));
          armed[st] = it + 1;
        }
      }
      if (!__shfl_sync(0xffffffffu, go, 0)) break;
    }
    // Never leave a copy in flight: wait for the last load of every stage.
    if (lane == 0) {
      for (int s = 0; s < C::kStages; ++s) {
        if (armed[s]) mbar_wait(&full[s], ((armed[s] - 1) / C::kStages) & 1);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdescY = idesc_bf16_f32(128, D);
      constexpr uint32_t kIdescP = (1u << 4) | (static_cast<uint32_t>(D >> 3) << 17) | (static_cast<uint32_t>(128 >> 4) << 24);
      const uint64_t pi_desc0 = desc_k_sw128(smem_u32(pi_s)), s_desc0 = desc_k_sw128(smem_u32(s_s)),
                     x_desc0 = desc_k_sw128(smem_u32(x_s));
      auto issue_y = [&](int it, int pslot) {
        const int st = it % C::kStages;
        const int b = it & 1;
        const uint32_t d_tmem = tmem + b * C::kSlotCols;
        const uint64_t xa = x_desc0 + static_cast<uint64_t>((st * C::kTileBytes) >> 4);
        // Small split first: the fp32 accumulator then rounds at the scale of
        // the large terms only during the last K-steps.
#pragma unroll
        for (int q = 0; q < 3; ++q) {
          const int sp = 2 - q;
#pragma unroll
          for (int k = 0; k < C::kKSteps; ++k) {
            constexpr int kAtomA = 128 * 128, kAtomB = D * 128;
            const uint64_t ad = xa + static_cast<uint64_t>(((k >> 2) * kAtomA + (k & 3) * 32) >> 4);
            const uint64_t bd = pi_desc0 + static_cast<uint64_t>(
                                               (pslot * C::kPiSlot + sp * C::kMatBytes + (k >> 2) * kAtomB + (k & 3) * 32) >> 4);
            umma_ss(d_tmem, ad, bd, kIdescY, (q | k) != 0);
          }
        }
        umma_commit(&yfull[b]);
        umma_commit(&empty[st]);        // the X stage is free once Y is computed
      };
      auto issue_p = [&](int it) {
        const int b = it & 1;
        const uint32_t slot = tmem + b * C::kSlotCols;
        // (A, B) pairs, small terms first: R2 S1, R1 S2, R1 S1.
#pragma unroll
        for (int pr = 0; pr < 3; ++pr) {
          const uint32_t acol = (pr == 0) ? C::kColR2 : C::kColR1;
          const int boff = (pr == 1) ? C::kMatBytes : 0;
#pragma unroll
          for (int k = 0; k < C::kKSteps; ++k) {
            constexpr int kAtomB = D * 128;
            const uint64_t bd = s_desc0 + static_cast<uint64_t>((boff + (k >> 2) * kAtomB + (k & 3) * 32) >> 4);
            umma_ts(slot, slot + acol + k * 8, bd, kIdescP, (pr | k) != 0);   // kind::f16, f16 A/B per kIdescP
          }
        }
        umma_commit(&pfull[b]);
      };
      int ny = 0, np = 0;
      int64_t icur = -1;                         // per-head mode: head of the last issued tile
      int inh = 0;                               // heads issued so far
      uint64_t last = globaltimer_ns();
      while (KEY ? (np < my_tiles) : (ny < my_tiles)) {
        if (*abort_s) break;
        bool progress = false;
        if (ny < my_tiles) {
          const int st = ny % C::kStages;
          const uint32_t ph = (ny / C::kStages) & 1;
          const uint32_t bph = (ny >> 1) & 1;
          const int64_t h = head_of(tile_of(ny));
          const int nh_t = (PH && h != icur) ? inh + 1 : inh;   // heads including this tile's
          const int pslot = PH ? (nh_t - 1) & 1 : 0;
          const bool pi_ok = !PH || h == icur || mbar_try_wait(&pi_full[pslot], ((nh_t - 1) >> 1) & 1);
          if (pi_ok && mbar_try_wait(&full[st], ph) && mbar_try_wait(&accfree[ny & 1], bph ^ 1)) {
            tc_fence_after();
            issue_y(ny, pslot);
            if (PH) {
              icur = h;
              inh = nh_t;
              // The head's last tile: its Pi slot is free once these MMAs complete.
              if (ny + 1 == my_tiles || head_of(tile_of(ny + 1)) != h) umma_commit(&pi_free[pslot]);
            }
            ++ny;
            progress = true;
          }
        }
        if (KEY && np < ny && mbar_try_wait(&rfull[np & 1], (np >> 1) & 1)) {
          tc_fence_after();
          issue_p(np);
          ++np;
          progress = true;
        }
        if (progress) {
          last = globaltimer_ns();
        } else {
          __nanosleep(32);              // nothing ready: leave the issue slots to the other warps
          if (globaltimer_ns() - last > a.wait_ns) {
            fail();
            break;
          }
        }
      }
    }
  } else {
    // --------------------------------------------------------------- epilogue
    const int wg = (warp - 2) >> 2;          // 0 or 1: tiles it with it % 2 == wg
    const int q = warp & 3;                  // TMEM lane quadrant of this warp
    const int row = q * 32 + lane;           // row within the tile
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(q * 32) << 16) + wg * C::kSlotCols;
    const int rshift = *rshift_s;
    const bool sym = *sym_s != 0;
    float th[kNb];
    for (int it = wg; it < my_tiles; it += 2) {
      const int64_t t = tile_of(it);
      const uint32_t ph = (it >> 1) & 1;
      const int64_t v = t * C::kM + row;
      const bool valid = v < a.n;
      if (!__all_sync(0xffffffffu, mbar_wait(&yfull[wg], ph, a.wait_ns))) {
        if (lane == 0) fail();
        break;
      }
      tc_fence_after();
      // Pass 1: ||y||^2, one 32-column chunk per wait (the loop is not
      // unrolled across chunks, which keeps the epilogue in the i-cache).
      float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
#pragma unroll 1
      for (int ch = 0; ch < C::kChunks; ++ch) {
        uint32_t yb[32];
        tmem_ld32(lane_addr + ch * 32, yb);
        tmem_ld_wait();
#pragma unroll
        for (int k = 0; k < 32; k += 4) {
          const float y0 = __uint_as_float(yb[k]), y1 = __uint_as_float(yb[k + 1]);
          const float y2 = __uint_as_float(yb[k + 2]), y3 = __uint_as_float(yb[k + 3]);
          s0 = fmaf(y0, y0, s0);
          s1 = fmaf(y1, y1, s1);
          s2 = fmaf(y2, y2, s2);
          s3 = fmaf(y3, y3, s3);
        }
      }
      const float nrm = sqrtf((s0 + s1) + (s2 + s3));
      const float band = kCodeGuard * nrm;
#pragma unroll
      for (int j = 0; j < kNb; ++j) th[j] = nrm > 0.f ? nrm * bnd_s[j] : bnd_s[j];
      // fp16 scale of r: 2^(13 - e - rshift) with nrm = m 2^e, m in [0.5, 1).
      float rscale = 1.f;
      if (KEY) {
        const int ex = static_cast<int>((__float_as_uint(nrm) >> 23) & 0xFFu);
        if (ex != 0) {
          int be = 266 - ex - rshift;
          be = be < 1 ? 1 : (be > 254 ? 254 : be);
          rscale = __uint_as_float(static_cast<uint32_t>(be) << 23);
        }
      }
      bool rowflag = false;                  // any coordinate or sign near its decision
      float rsq = 0.f;
      uint8_t* dst = a.idx + v * kRowBytes;
      // Pass 2, per chunk: codes (stored as the chunk's BITS words), and for
      // keys the fp16 splits of r 2^k into TMEM.
      // The symmetric-codebook search (3 bits) runs when the table allows it;
      // both loops are compiled, one runs per CTA.
      auto pass2 = [&](auto sym_tag) {
        constexpr bool SYM = decltype(sym_tag)::value;
  #pragma unroll 1
        for (int ch = 0; ch < C::kChunks; ++ch) {
          uint32_t yb[32];
          tmem_ld32(lane_addr + ch * 32, yb);
          tmem_ld_wait();
          uint32_t cw[BITS];
  #pragma unroll
          for (int w = 0; w < BITS; ++w) cw[w] = 0u;
          uint32_t r1[16], r2[16];
  #pragma unroll
          for (int k = 0; k < 32; k += 2) {
            float rr[2];
  #pragma unroll
            for (int e = 0; e < 2; ++e) {
              const float y = __uint_as_float(yb[k + e]);
              int c;
              if constexpr (SYM) c = code_symmetric3(y, th, band, rowflag);
              else c = code_guarded<BITS>(y, th, band, rowflag);
              const int bp = (k + e) * BITS;
              cw[bp >> 5] |= static_cast<uint32_t>(c) << (bp & 31);
              if ((bp & 31) + BITS > 32) cw[(bp >> 5) + 1] |= static_cast<uint32_t>(c) >> (32 - (bp & 31));
              rr[e] = KEY ? fmaf(-nrm, cent_s[c], y) : 0.f;
            }
            if (KEY) {
              rsq = fmaf(rr[0], rr[0], fmaf(rr[1], rr[1], rsq));
              const float a0 = rr[0] * rscale, a1 = rr[1] * rscale;
              const __half2 h = __floats2half2_rn(a0, a1);
              const float2 hf = __half22float2(h);
              const __half2 l = __floats2half2_rn(a0 - hf.x, a1 - hf.y);
              r1[k / 2] = *reinterpret_cast<const uint32_t*>(&h);
              r2[k / 2] = *reinterpret_cast<const uint32_t*>(&l);
            }
          }
          if (KEY) {
            tmem_st16(lane_addr + C::kColR1 + ch * 16, r1);
            tmem_st16(lane_addr + C::kColR2 + ch * 16, r2);
          }
          if (valid) {
            // The chunk's 4 BITS bytes at byte 4 BITS ch of the row.
            uint32_t* cdst = reinterpret_cast<uint32_t*>(dst + ch * 4 * BITS);
            if constexpr (BITS == 4) {
              reinterpret_cast<uint4*>(cdst)[0] = make_uint4(cw[0], cw[1], cw[2], cw[3]);
            } else if constexpr (BITS == 2) {
              reinterpret_cast<uint2*>(cdst)[0] = make_uint2(cw[0], cw[1]);
            } else {
  #pragma unroll
              for (int w = 0; w < BITS; ++w) cdst[w] = cw[w];
            }
          }
        }
      };
      if (BITS == 3 && sym) pass2(std::integral_constant<bool, BITS == 3>{});
      else pass2(std::false_type{});
      if (!KEY) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&accfree[wg]);
        // Values: a row with an undecided code is flagged by the sign bit of
        // its norm; quantize_fixup redoes it.
        if (valid) a.norm[v] = rowflag ? -nrm : nrm;
      } else {
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&rfull[wg]);
        if (valid) a.norm[v] = nrm;
        const float rn = sqrtf(rsq);
        const float sband = kSignGuard * rn * rscale;
        if (!__all_sync(0xffffffffu, mbar_wait(&pfull[wg], ph, a.wait_ns))) {
          if (lane == 0) fail();
          break;
        }
        tc_fence_after();
#pragma unroll 1
        for (int ch = 0; ch < C::kChunks; ++ch) {
          uint32_t pb[32];
          tmem_ld32(lane_addr + ch * 32, pb);
          tmem_ld_wait();
          uint32_t word = 0;
          bool near = false;
#pragma unroll
          for (int k = 0; k < 32; ++k) {
            const float p = __uint_as_float(pb[k]);
            word |= (p >= 0.f ? 1u : 0u) << k;
            near |= fabsf(p) < sband;
          }
          rowflag |= near;
          if (valid) a.sign[v * C::kChunks + ch] = word;
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&accfree[wg]);
        if (valid) a.rnorm[v] = rowflag ? __uint_as_float(__float_as_uint(rn) | 0x80000000u) : rn;
      }
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

// ---------------------------------------------------------------------------
// Exact recomputation of flagged rows (fp64). The flag is the sign bit of the
// row's stored ||r|| (keys) or ||x|| (values); every output of the row is
// rewritten and the flag cleared. One CTA per SM scans a contiguous range of
// rows into a shared-memory list; if the list is not empty it stages Pi^T (and
// S^T) in shared memory, fp32, laid out so that lane l reads the G = D/32
// entries of its output coordinates l, l + 32, ... for one input coordinate
// with one 16-byte (8-byte for d = 64) load. A warp takes kFixBatch rows at a
// time: the x (later r) of the rows sit in the warp's fp64 scratch and are
// read as broadcasts; every converted matrix entry serves all rows of the batch.
// ---------------------------------------------------------------------------
constexpr int kFixThreads = 512;       // 16 warps
constexpr int kFixWarps = kFixThreads / 32;
constexpr int kFixList = 16384;        // rows scanned per round (list capacity; one
                                       // round covers a CTA's share of a 2M-row call)
constexpr int kFixBatch = 4;           // rows per warp at a time
constexpr int kFixGridRows = 8192;     // rows per fixup CTA when the call is smaller than the grid

template <int D, bool KEY>
struct FixCfg {
  static constexpr size_t kMat = sizeof(float) * size_t(D) * D;
  static constexpr size_t kOffS = kMat;
  static constexpr size_t kOffScr = kOffS + (KEY ? kMat : 0);
  static constexpr size_t kScr = sizeof(double) * size_t(kFixBatch) * D;  // per warp
  static constexpr size_t kOffList = kOffScr + kScr * kFixWarps;
  static constexpr size_t kBytes = kOffList + sizeof(uint16_t) * kFixList;
};

// M^T staged as [k][lane][c] = M[32 c + lane][k]. The lanes of a warp read 16
// bytes each from consecutive rows of M and write with stride G words.
template <int D>
__device__ __forceinline__ void stage_transposed(float* dst, const float* __restrict__ M) {
  constexpr int G = D / 32;
  constexpr int kIt = D * D / 4 / kFixThreads;   // loads per thread, all in flight at once
  static_assert(kIt * kFixThreads * 4 == D * D, "staging covers the matrix");
  // Every CTA starts at a different part of the matrix, so the SMs do not all
  // read the same L2 lines at once.
  const int rot = static_cast<int>(blockIdx.x % kIt);
  float4 f[kIt];
#pragma unroll
  for (int it = 0; it < kIt; ++it) {
    const int e = threadIdx.x + ((it + rot) % kIt) * kFixThreads;
    f[it] = __ldg(reinterpret_cast<const float4*>(M + (e % D) * D) + e / D);
  }
#pragma unroll
  for (int it = 0; it < kIt; ++it) {
    const int e = threadIdx.x + ((it + rot) % kIt) * kFixThreads;
    const int i = e % D, k4 = e / D;
    const int l = i & 31, c = i >> 5;
    dst[((4 * k4 + 0) * 32 + l) * G + c] = f[it].x;
    dst[((4 * k4 + 1) * 32 + l) * G + c] = f[it].y;
    dst[((4 * k4 + 2) * 32 + l) * G + c] = f[it].z;
    dst[((4 * k4 + 3) * 32 + l) * G + c] = f[it].w;
  }
}

// out[r][c] = sum_k M[32 c + lane][k] v_r[k] for the n rows of the batch, fp64.
template <int D>
__device__ __forceinline__ void batch_matvec(const float* MT, const double* scr, int n,
                                             double (&out)[kFixBatch][D / 32]) {
  constexpr int G = D / 32;
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int r = 0; r < kFixBatch; ++r)
#pragma unroll
    for (int c = 0; c < G; ++c) out[r][c] = 0.0;
  // Blocks of four input coordinates: every load of a block is issued before
  // its arithmetic. Rows r >= n of the scratch hold stale values; their
  // results are discarded by the caller.
  (void)n;
#pragma unroll 2
  for (int k0 = 0; k0 < D; k0 += 4) {
    float wf[4][G];
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      if constexpr (G == 4) {
        const float4 f = reinterpret_cast<const float4*>(MT)[(k0 + kk) * 32 + lane];
        wf[kk][0] = f.x; wf[kk][1] = f.y; wf[kk][2] = f.z; wf[kk][3] = f.w;
      } else {
        const float2 f = reinterpret_cast<const float2*>(MT)[(k0 + kk) * 32 + lane];
        wf[kk][0] = f.x; wf[kk][1] = f.y;
      }
    }
    double v[kFixBatch][4];
#pragma unroll
    for (int r = 0; r < kFixBatch; ++r) {
      const double2 a = reinterpret_cast<const double2*>(scr + r * D + k0)[0];
      const double2 b = reinterpret_cast<const double2*>(scr + r * D + k0)[1];
      v[r][0] = a.x; v[r][1] = a.y; v[r][2] = b.x; v[r][3] = b.y;
    }
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
      for (int c = 0; c < G; ++c) {
        const double w = wf[kk][c];
#pragma unroll
        for (int r = 0; r < kFixBatch; ++r) out[r][c] = fma(w, v[r][kk], out[r][c]);
      }
    }
  }
}

template <int D, bool KEY, int BITS>
__device__ __forceinline__ void fix_batch(const TcArgs& a, const int64_t (&rows)[kFixBatch], int n, const float* PiT,
                                          const float* ST, double* scr, const float* cent, const float* bnd) {
  constexpr int kNb = (1 << BITS) - 1;
  constexpr int G = D / 32;
  const int lane = threadIdx.x & 31;
  // x of every row as fp64 into the scratch, and ||x||. The loads of all rows
  // are issued before any arithmetic; rows r >= n repeat row 0 (a valid
  // address) and their values are not used.
  double n64[kFixBatch];
  float xf[kFixBatch][G];
#pragma unroll
  for (int r = 0; r < kFixBatch; ++r) {
    const __nv_bfloat16* xr = a.x + rows[r] * a.row_stride;
#pragma unroll
    for (int c = 0; c < G; ++c) xf[r][c] = __bfloat162float(xr[32 * c + lane]);
  }
#pragma unroll
  for (int r = 0; r < kFixBatch; ++r) {
    double nn = 0.0;
#pragma unroll
    for (int c = 0; c < G; ++c) {
      const double xv = static_cast<double>(xf[r][c]);
      scr[r * D + 32 * c + lane] = xv;
      nn = fma(xv, xv, nn);
    }
    n64[r] = r < n ? sqrt(warp_sum(nn)) : 0.0;
  }
  __syncwarp();
  double y[kFixBatch][G];
  batch_matvec<D>(PiT, scr, n, y);
  __syncwarp();                                          // x is dead: the scratch takes r
#pragma unroll
  for (int r = 0; r < kFixBatch; ++r) {
    if (r >= n) continue;
    uint32_t* idx = reinterpret_cast<uint32_t*>(a.idx + rows[r] * (D * BITS / 8));
    double rr = 0.0;
#pragma unroll
    for (int c = 0; c < G; ++c) {
      const uint32_t code = static_cast<uint32_t>(exact_code<kNb>(y[r][c], n64[r], bnd));
      if (KEY) {
        const double res = y[r][c] - n64[r] * static_cast<double>(cent[code]);
        scr[r * D + 32 * c + lane] = res;
        rr = fma(res, res, rr);
      }
      // Coordinates 32 c .. 32 c + 31 fill packed words c BITS .. c BITS + BITS - 1.
      const int o = BITS * lane;
#pragma unroll
      for (int w = 0; w < BITS; ++w) {
        uint32_t val = 0u;
        if ((o >> 5) == w) val |= code << (o & 31);
        if ((o >> 5) == w - 1 && (o & 31) + BITS > 32) val |= code >> (32 - (o & 31));
        const uint32_t word = __reduce_or_sync(0xffffffffu, val);
        if (lane == w) idx[c * BITS + w] = word;
      }
    }
    if (lane == 0) a.norm[rows[r]] = static_cast<float>(n64[r]);
    if (KEY) {
      const double rn = sqrt(warp_sum(rr));
      if (lane == 0) a.rnorm[rows[r]] = static_cast<float>(rn);
    }
  }
  if (KEY) {
    __syncwarp();
    double pv[kFixBatch][G];
    batch_matvec<D>(ST, scr, n, pv);
#pragma unroll
    for (int r = 0; r < kFixBatch; ++r) {
      if (r >= n) continue;
#pragma unroll
      for (int c = 0; c < G; ++c) {
        const uint32_t word = __ballot_sync(0xffffffffu, pv[r][c] >= 0.0);
        if (lane == c) a.sign[rows[r] * G + c] = word;
      }
    }
  }
  __syncwarp();                                          // scratch reused by the next batch
}

// Per-head mode: a window never crosses a head, and Pi^T is staged again
// when a window with flagged rows belongs to another head than the last.
template <int D, bool KEY, int BITS, bool PH>
__global__ void __launch_bounds__(kFixThreads, 1) quantize_fixup(TcArgs a) {
  using F = FixCfg<D, KEY>;
  extern __shared__ __align__(16) unsigned char fix_smem[];
  float* PiT = reinterpret_cast<float*>(fix_smem);
  float* ST = reinterpret_cast<float*>(fix_smem + F::kOffS);
  uint16_t* list = reinterpret_cast<uint16_t*>(fix_smem + F::kOffList);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  double* scr = reinterpret_cast<double*>(fix_smem + F::kOffScr + F::kScr * warp);
  __shared__ float cent_s[16], bnd_s[16];
  __shared__ int cnt, taken;
  if (threadIdx.x < 16) {
    cent_s[threadIdx.x] = threadIdx.x <= (1 << BITS) - 1 ? a.cent[threadIdx.x] : 0.f;
    bnd_s[threadIdx.x] = threadIdx.x < (1 << BITS) - 1 ? a.bnd[threadIdx.x] : 0.f;
  }
  const float* flagp = KEY ? a.rnorm : a.norm;
  const int64_t per = (a.n + gridDim.x - 1) / gridDim.x;
  const int64_t r0 = int64_t(blockIdx.x) * per;
  const int64_t r1 = r0 + per < a.n ? r0 + per : a.n;
  bool staged = false;
  int64_t staged_head = -1;
  int64_t w1 = r0;
  for (int64_t w0 = r0; w0 < r1; w0 = w1) {
    w1 = w0 + kFixList < r1 ? w0 + kFixList : r1;
    if (PH) {
      const int64_t hb = (w0 / a.vpp + 1) * a.vpp;          // next head boundary
      if (hb < w1) w1 = hb;
    }
    if (threadIdx.x == 0) {
      cnt = 0;
      taken = 0;
    }
    __syncthreads();
    // Scan: every thread loads its flag words of the window first
    // (independent loads), then records the flagged rows.
    {
      constexpr int kPer = kFixList / kFixThreads;       // rows per thread per window
      uint32_t fw[kPer];
#pragma unroll
      for (int u = 0; u < kPer; ++u) {
        const int64_t row = w0 + threadIdx.x + int64_t(u) * kFixThreads;
        fw[u] = row < w1 ? __float_as_uint(__ldg(flagp + row)) : 0u;
      }
#pragma unroll
      for (int u = 0; u < kPer; ++u)
        if (fw[u] >> 31) list[atomicAdd(&cnt, 1)] = static_cast<uint16_t>(threadIdx.x + u * kFixThreads);
    }
    __syncthreads();
    const int total = cnt;
    if (total == 0) continue;
    const int64_t head = PH ? w0 / a.vpp : 0;
    if (!staged || head != staged_head) {
      stage_transposed<D>(PiT, a.Pi + head * a.pi_stride);
      if (KEY && !staged) stage_transposed<D>(ST, a.S);
      __syncthreads();
      staged = true;
      staged_head = head;
    }
    for (;;) {
      int e = 0;
      if (lane == 0) e = atomicAdd(&taken, kFixBatch);
      e = __shfl_sync(0xffffffffu, e, 0);
      if (e >= total) break;
      const int n = total - e < kFixBatch ? total - e : kFixBatch;
      int64_t rows[kFixBatch];
#pragma unroll
      for (int r = 0; r < kFixBatch; ++r) rows[r] = w0 + list[e + (r < n ? r : 0)];
      fix_batch<D, KEY, BITS>(a, rows, n, PiT, ST, scr, cent_s, bnd_s);
    }
    __syncthreads();
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

template <int D, bool KEY, int BITS, bool PH>
cudaError_t launch_tc(const TcArgs& a, const CUtensorMap& map, cudaStream_t st) {
  using C = Cfg<D, KEY, PH>;
  static_assert(C::kSmemBytes <= 232448, "shared memory plan exceeds 227 KB");
  cudaError_t e = cudaFuncSetAttribute(quantize_tc_kernel<D, KEY, BITS, PH>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t tiles = (a.n + 127) / 128;
  const int grid = static_cast<int>(tiles < sms ? tiles : sms);
  quantize_tc_kernel<D, KEY, BITS, PH><<<grid, kThreads, C::kSmemBytes, st>>>(map, a);
  count_launch();
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  constexpr size_t fix_smem = FixCfg<D, KEY>::kBytes;
  static_assert(FixCfg<D, KEY>::kBytes <= 232448, "fixup shared memory plan exceeds 227 KB");
  e = cudaFuncSetAttribute(quantize_fixup<D, KEY, BITS, PH>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(fix_smem));
  if (e != cudaSuccess) return e;
  // One CTA per 8,192 rows, at most one per SM (a CTA's share then fits one
  // scan window up to 148 x 16,384 rows).
  const int64_t fix_ctas = (a.n + kFixGridRows - 1) / kFixGridRows;
  quantize_fixup<D, KEY, BITS, PH><<<static_cast<int>(fix_ctas < sms ? (fix_ctas < 1 ? 1 : fix_ctas) : sms),
                                     kFixThreads, fix_smem, st>>>(a);
  count_launch();
  return cudaGetLastError();
}

template <int D, bool KEY, bool PH = false>
cudaError_t launch_bits(int bits, const TcArgs& a, const CUtensorMap& map, cudaStream_t st) {
  switch (bits) {
    case 2: return launch_tc<D, KEY, 2, PH>(a, map, st);
    case 3: return launch_tc<D, KEY, 3, PH>(a, map, st);
    default: return launch_tc<D, KEY, 4, PH>(a, map, st);
  }
}

}  // namespace

bool tc_quantize_supported(int d, int x_dtype, bool rope, int64_t vectors_per_pi, int64_t pi_stride, const void* x,
                           int64_t row_stride) {
  if (!(d == 64 || d == 128)) return false;
  if (x_dtype != TQ_BF16 || rope) return false;
  // Per-head rotations: d = 64 (two Pi slots fit beside the pipeline), and no
  // 128-vector tile may straddle two heads.
  if (pi_stride != 0 && !(d == 64 && vectors_per_pi > 0 && vectors_per_pi % 128 == 0)) return false;
  if (!aligned(x, 16) || (row_stride * 2) % 16 != 0) return false;
  return encode_fn() != nullptr;
}

tq_status tc_quantize(int d, bool is_key, int bits, const void* x, int64_t n, int64_t row_stride, const float* Pi,
                      int64_t vectors_per_pi, int64_t pi_stride, const float* S, const float* cent, const float* bnd,
                      const tq_planes* out, int32_t* d_status, cudaStream_t st) {
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
           is_key ? out->sign : nullptr, out->norm, is_key ? out->rnorm : nullptr, d_status, pipeline_wait_ns(),
           pi_stride != 0 ? vectors_per_pi : 1, pi_stride};
  cudaError_t e;
  if (d == 128)
    e = is_key ? launch_bits<128, true>(bits, a, map, st) : launch_bits<128, false>(bits, a, map, st);
  else if (pi_stride != 0)
    e = is_key ? launch_bits<64, true, true>(bits, a, map, st) : launch_bits<64, false, true>(bits, a, map, st);
  else
    e = is_key ? launch_bits<64, true>(bits, a, map, st) : launch_bits<64, false>(bits, a, map, st);
  if (e != cudaSuccess) return fail(TQ_ERR_CUDA, "tensor-core quantize launch: %s", cudaGetErrorString(e));
  return TQ_OK;
}

}  // namespace tq
