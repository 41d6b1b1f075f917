// Tensor-core decode attention (sm_100a, tcgen05 kind::i8) for d = 128 with
// four query rows per KV stream (the GQA decode shape) and 3-bit values.
//
// Sources: gist.science "TurboESM ..." section 2E (one fused kernel unpacks
// the codes, applies the QJL correction and the inverse rotation and runs an
// online softmax, with no dequantised tensor in memory) and 7minutos.es
// "KV cache ... TurboQuant" Etapa 2 (the QJL estimator).
//
// Both contractions of decode run on the tensor cores over operands rebuilt
// from the packed cache in on-chip memory, with exact integer arithmetic:
//   scores  A (TMEM, one lane per token), 128 columns per tile:
//             a1 | a2 | a3   the key codebook value of every coordinate as
//                            three int8 limbs, c = sc (a1 + a2/128 + a3/128^2)
//             sgn            the sign bits, masked in place: byte 16 j + b is
//                            byte b of the sign row AND (1 << j), i.e. bit
//                            8 b + j of the sketch times 2^j (unsigned)
//           B (smem, K-major): per query row four int8 limbs of q_rot and of
//           s' = s 2^-(i mod 8) (sign-chunk rows permuted to match). Limb
//           products of equal weight 128^-w go to the same int32 column: the
//           a1, a2, a3 chunks use B tiles whose limb columns are shifted by
//           0, 1, 2, so D column 4 r + w holds sum_{l+m=w} a_l q_m.
//   values  O[i][n] = sum_t c_V[code_ti] w_t,n: A (smem, M-major) the value
//           codebook as two int8 limbs per coordinate, one 128-byte row per
//           token; B the tile's weights w = p ||v|| / s_item as three int8
//           limbs per query row, s_item = max ||v|| over the work item / 127
//           (p <= 1 because the running maximum only grows).
// Online softmax: the running maximum per row only moves when a score of the
// tile exceeds it (a vote over the softmax warps; the tile maximum is reduced
// only then), so an ordinary tile costs one barrier; l is kept per thread and
// summed once per work item. The value warps fold each PV product into their
// accumulators (thread = coordinate) with the tile's correction, which the
// softmax warps leave in a four-slot ring.
// Roles (480 threads, one persistent CTA per SM):
//   warp 0     bulk copies of the packed index / sign planes into a 3-stage ring
//   warp 1     TMEM owner and single-thread issuer of the score MMAs
//   warp 14    single-thread issuer of the PV MMAs
//   warps 2-5  key operand generation into TMEM        (thread = token)
//   warps 6-9  value operand generation into smem      (thread = token)
//             and the value epilogue                   (thread = coordinate)
//   warps 10-13 scores, softmax and weight limbs       (thread = token); the
//             even and odd tiles of a work item keep separate running maxima
//             and sums, so a work item leaves two partial records
// Every wait is bounded (2 s); a timeout sets TQ_DEV_TIMEOUT and the CTA
// drains its copies and MMAs before it frees TMEM and returns.
#include <cuda.h>
#include <cuda_runtime.h>

#include "tq_decode_tc.h"
#include "tq_device.cuh"
#include "tq_internal.h"
#include "tq_sm100.cuh"

namespace tq {
namespace {

using namespace sm100;
using dev::warp_max;
using dev::warp_sum;

constexpr int kD = 128;
constexpr int kTT = 128;               // tokens per tile
constexpr int kStages = 3;
constexpr int kThreadsTc = 480;        // 15 warps
constexpr int kRowsTc = 4;

// TMEM columns (32-bit): A_score x2 at 0, 128 (a1 | a2 | a3 | sgn, 32 each);
// D_score x2 at 256, 288 (mse 16 | sgn 16); D_o x2 at 320, 352 (limb chains).
constexpr uint32_t kColA = 0, kColDs = 256, kColDo = 320, kTmemColsTc = 512;

// Instruction descriptor, kind::i8: s32 D, M = 128, N = 16.
__host__ __device__ constexpr uint32_t idesc_i8(bool a_signed, bool a_mn_major) {
  return (2u << 4) | ((a_signed ? 1u : 0u) << 7) | (1u << 10) | ((a_mn_major ? 1u : 0u) << 15) |
         ((16u >> 3) << 17) | ((128u >> 4) << 24);
}

template <int KB>
struct TcSm {
  static constexpr int kRbk = kD * KB / 8;
  static constexpr int kStageBytes = kTT * (kRbk + 16 + 48);       // kidx | ksign | vidx
  static constexpr int kStageStride = ((kStageBytes + 1023) / 1024) * 1024;
  static constexpr int kOffVh = kStages * kStageStride;            // 1024-aligned
  static constexpr int kVhBytes = 2 * kTT * 128;                    // two limbs x 128 tokens x 128 B
  static constexpr int kOffP = kOffVh + 2 * kVhBytes;               // 2 x [16 rows x 128 B]
  static constexpr int kOffB = kOffP + 2 * 2048;                    // 2 items x (B1 | B2 | B3 | Bs)
  static constexpr int kOffBar = kOffB + 2 * 4 * 2048;
  static constexpr int kNumBars = 2 * kStages + 2 * 11 + 2;
  static constexpr int kOffMisc = ((kOffBar + kNumBars * 8 + 15) / 16) * 16;
  static constexpr int kOffRing = kOffMisc + 16;                    // [4 tiles][8]: corr[4], scale
  static constexpr int kOffRed = kOffRing + 4 * 8 * 4;              // [2 groups][4 warps][16]
  static constexpr int kOffRed2 = kOffRed + 2 * 4 * 16 * 4;         // [2 groups][4 warps][4]
  static constexpr int kOffTab = kOffRed2 + 2 * 4 * 4 * 4;          // ka1 ka2 ka3 va1 va2 (4 words) + 2 scales
  static constexpr int kBytes = kOffTab + 22 * 4 + 1024;
};

struct TcDecodeArgs {
  DecodeArgs v;
  int n_items;
};

// int8 limbs of a codebook, c ~ scale (a1 + a2/128 + a3/128^2) with
// scale = max|c| / 127, as byte tables (byte k of word k/4 = code k); t3 may
// be null (two limbs). Computed in fp64 by one thread; every CTA derives the
// same tables.
__device__ void codebook_limbs(const float* c, int n, uint32_t* t1, uint32_t* t2, uint32_t* t3, float* scale) {
  double m = 0.0;
  for (int k = 0; k < n; ++k) m = fmax(m, fabs(static_cast<double>(__ldg(c + k))));
  const double sc = m > 0.0 ? m / 127.0 : 1.0;
  for (int w = 0; w < 4; ++w) {
    t1[w] = t2[w] = 0u;
    if (t3) t3[w] = 0u;
  }
  auto put = [](uint32_t* t, int k, double v) {
    t[k / 4] |= static_cast<uint32_t>(static_cast<uint8_t>(static_cast<int8_t>(v))) << (8 * (k % 4));
  };
  for (int k = 0; k < n; ++k) {
    const double r0 = static_cast<double>(__ldg(c + k)) / sc;
    const double a1 = rint(r0);
    const double r1 = (r0 - a1) * 128.0;
    const double a2 = rint(r1);
    put(t1, k, a1);
    put(t2, k, a2);
    if (t3) put(t3, k, rint((r1 - a2) * 128.0));
  }
  *scale = static_cast<float>(sc);
}

__device__ __forceinline__ bool wg_sync_or(int id, bool p) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred pi, po;\n\t"
      "setp.ne.u32 pi, %1, 0;\n\t"
      "barrier.cta.red.or.pred po, %2, 128, pi;\n\t"
      "selp.u32 %0, 1, 0, po;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(p)), "r"(id)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ void wg_sync(int id) { asm volatile("bar.sync %0, 128;" ::"r"(id) : "memory"); }

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t s) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(s));
  return d;
}

// 8 three-bit codes (bits 0..23 of x; bits above ignored) -> one word of
// eight nibbles c0..c7; PRMT reads the low 16 bits as the selector of c0..c3.
// Each step moves the upper half of every field up by adding a multiple of
// it (no field carries into the next).
__device__ __forceinline__ uint32_t nibbles3(uint32_t x) {
  const uint32_t y = ((x & 0xFFF000u) << 4) | (x & 0xFFFu);            // c0-3 | c4-7 in halves
  const uint32_t z = y + 3u * (y & 0x0FC00FC0u);                       // two codes per byte
  return z + (z & 0x38383838u);                                        // one code per nibble
}
// 8 two-bit codes (bits 0..15 of x) -> eight nibbles.
__device__ __forceinline__ uint32_t nibbles2(uint32_t x) {
  const uint32_t y = ((x & 0xFF00u) << 8) | (x & 0xFFu);
  const uint32_t z = y + 15u * (y & 0x00F000F0u);
  return z + 3u * (z & 0x0C0C0C0Cu);
}
// Byte lookup of four codes in a 16-entry table given as four words (codes
// 0-3 | 4-7 | 8-11 | 12-15); `nib` holds the four 4-bit codes.
__device__ __forceinline__ uint32_t lut16(const uint32_t (&t)[4], uint32_t nib) {
  const uint32_t s = nib & 0x7777u;
  const uint32_t lo = prmt(t[0], t[1], s), hi = prmt(t[2], t[3], s);
  // byte k takes `hi` when bit 3 of nibble k is set
  const uint32_t m8 = (nib >> 3) & 0x1111u;
  const uint32_t mk = prmt(m8 * 0xFu, 0u, 0x3210u);   // nibbles 0/F in the low 16 bits
  const uint32_t mask = ((mk & 0xFu) ? 0xFFu : 0u) | ((mk & 0xF0u) ? 0xFF00u : 0u) | ((mk & 0xF00u) ? 0xFF0000u : 0u) |
                        ((mk & 0xF000u) ? 0xFF000000u : 0u);
  return (lo & ~mask) | (hi & mask);
}

__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void umma_i8_ss(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}
__device__ __forceinline__ void umma_i8_ts(uint32_t d, uint32_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d),
      "r"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}
// Swizzled byte offset (128-byte rows, 8-row 1024-byte atoms) of byte k of row r.
__device__ __forceinline__ uint32_t sw_byte(int r, int k) {
  return static_cast<uint32_t>(r * 128 + ((((k >> 4) ^ (r & 7))) << 4) + (k & 15));
}
// Four int8 limbs of x (|x| <= 127): x ~ l0 + l1/128 + l2/128^2 + l3/128^3.
__device__ __forceinline__ void limbs4(float x, int (&l)[4]) {
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    l[u] = __float2int_rn(x);
    x = (x - static_cast<float>(l[u])) * 128.f;
  }
}
// int32 accumulator -> float (exact: every accumulator here stays below 2^22,
// at most 3 limb products of 128 terms with limbs <= 127 in magnitude).
__device__ __forceinline__ float i2f(uint32_t x) { return static_cast<float>(static_cast<int32_t>(x)); }
__device__ __forceinline__ float limb_sum4(const uint32_t* d) {
  float v = i2f(d[3]);
  v = fmaf(v, 1.f / 128.f, i2f(d[2]));
  v = fmaf(v, 1.f / 128.f, i2f(d[1]));
  return fmaf(v, 1.f / 128.f, i2f(d[0]));
}
__device__ __forceinline__ float limb_sum3(const uint32_t* d) {
  return fmaf(fmaf(i2f(d[2]), 1.f / 128.f, i2f(d[1])), 1.f / 128.f, i2f(d[0]));
}
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <int KB>
__global__ void __launch_bounds__(kThreadsTc, 1) decode_tc_kernel(TcDecodeArgs A) {
  using Sm = TcSm<KB>;
  constexpr int kRbk = Sm::kRbk;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const DecodeArgs& a = A.v;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + Sm::kOffBar);
  uint64_t* st_full = bars;                       // [3]
  uint64_t* st_empty = bars + kStages;            // [3]
  uint64_t* a_full = bars + 2 * kStages;          // [2]
  uint64_t* a_free = a_full + 2;                  // [2] (aliased below)
  uint64_t* s_full = a_free + 2;                  // [2]
  uint64_t* ds_free = s_full + 2;                 // [2]
  uint64_t* vh_full = ds_free + 2;                // [2]
  uint64_t* vh_free = vh_full + 2;                // [2] (aliased below)
  uint64_t* p_full = vh_free + 2;                 // [2]
  uint64_t* p_free = p_full + 2;                  // [2] (aliased below)
  uint64_t* pv_full = p_free + 2;                 // [2]
  uint64_t* do_free = pv_full + 2;                // [2]
  uint64_t* b_full = do_free + 2;                 // [2] per item parity
  uint64_t* drain = b_full + 2;                   // [2] score issuer, PV issuer
  // One completion event each: the score MMAs of a tile free its key operands
  // and fill its score columns; the PV MMAs free the value operands and the
  // weight tile and fill the value columns.
  a_free = s_full;
  vh_free = pv_full;
  p_free = pv_full;
  uint32_t* tmem_base_s = reinterpret_cast<uint32_t*>(sm + Sm::kOffMisc);
  volatile int* abort_s = reinterpret_cast<volatile int*>(sm + Sm::kOffMisc + 4);
  float* ring = reinterpret_cast<float*>(sm + Sm::kOffRing);          // [4][8]
  float* red = reinterpret_cast<float*>(sm + Sm::kOffRed);            // [4 warps][16]
  float* red2 = reinterpret_cast<float*>(sm + Sm::kOffRed2);          // [4 warps][4]
  uint32_t* tab = reinterpret_cast<uint32_t*>(sm + Sm::kOffTab);      // ka1 ka2 ka3 va1 va2 (4 words each)
  float* cb_scale = reinterpret_cast<float*>(sm + Sm::kOffTab + 20 * 4);   // key, value codebook scales

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const DecodeShape& sh = a.sh;

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&st_full[s], 1);
      mbar_init(&st_empty[s], 8);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&a_full[b], 4);
      mbar_init(&a_free[b], 1);
      mbar_init(&s_full[b], 1);
      mbar_init(&ds_free[b], 4);
      mbar_init(&vh_full[b], 4);
      mbar_init(&vh_free[b], 1);
      mbar_init(&p_full[b], 4);
      mbar_init(&p_free[b], 1);
      mbar_init(&pv_full[b], 1);
      mbar_init(&do_free[b], 4);
      mbar_init(&b_full[b], 4);
    }
    mbar_init(&drain[0], 1);
    mbar_init(&drain[1], 1);
    *abort_s = 0;
    for (int k = 0; k < 4; ++k) reinterpret_cast<int*>(sm + Sm::kOffRing)[k * 8 + 5] = -1;
    mbar_fence_init();
  }
  if (tid == 32) {
    codebook_limbs(a.cK, 1 << sh.kbits, tab, tab + 4, tab + 8, &cb_scale[0]);
    codebook_limbs(a.cV, 8, tab + 12, tab + 16, nullptr, &cb_scale[1]);
  }
  if (warp == 1) {
    tmem_alloc(tmem_base_s, kTmemColsTc);
    tmem_relinquish();
  }
  // Rows 12-15 of both weight tiles stay zero (3 limbs x 4 rows are used).
  for (int e = tid; e < 2 * 512 / 16; e += kThreadsTc) {
    const int b = e / 32, o = e % 32;
    reinterpret_cast<uint4*>(sm + Sm::kOffP + b * 2048 + 1536)[o] = make_uint4(0u, 0u, 0u, 0u);
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_base_s;
  auto fail = [&]() {
    *abort_s = 1;
    if (a.d_status) atomicOr(a.d_status, TQ_DEV_TIMEOUT);
  };
  const float k_scale = cb_scale[0], v_scale = cb_scale[1];

  // Item sequence (identical in every role): items blockIdx.x, +gridDim.x, ...
  // item -> (unit, split); tiles of 128 tokens inside the split.
  auto item_tiles = [&](int item, int64_t& t_begin, int64_t& t_end) -> int {
    const int split = item % sh.n_splits;
    t_begin = int64_t(split) * sh.chunk;
    t_end = (t_begin + sh.chunk < sh.n_ctx) ? t_begin + sh.chunk : sh.n_ctx;
    return static_cast<int>((t_end - t_begin + kTT - 1) / kTT);
  };
  auto item_row0 = [&](int item) -> int64_t {
    const int64_t unit = item / sh.n_splits;       // row_blocks == 1 for this kernel
    return unit * sh.ctx_stride;
  };

  if (warp == 0) {
    // ------------------------------------------------------------- loader
    if (lane == 0) {
      int j = 0;
      bool ok = true;
      for (int item = blockIdx.x; ok && item < A.n_items; item += gridDim.x) {
        int64_t tb, te;
        const int nt_tiles = item_tiles(item, tb, te);
        const int64_t row0 = item_row0(item);
        for (int tj = 0; tj < nt_tiles; ++tj, ++j) {
          const int s = j % kStages;
          if (*abort_s || !mbar_wait(&st_empty[s], ((j / kStages) & 1) ^ 1)) { ok = false; break; }
          const int64_t t0 = tb + int64_t(tj) * kTT;
          const int nt = static_cast<int>((te - t0 < kTT) ? te - t0 : kTT);
          const uint32_t bk = nt * kRbk, bs = nt * 16, bv = nt * 48;
          mbar_expect_tx(&st_full[s], bk + bs + bv);
          unsigned char* st = sm + s * Sm::kStageStride;
          bulk_g2s(st, a.kidx + (row0 + t0) * kRbk, bk, &st_full[s]);
          bulk_g2s(st + kTT * kRbk, a.ksign + (row0 + t0) * 4, bs, &st_full[s]);
          bulk_g2s(st + kTT * (kRbk + 16), a.vidx + (row0 + t0) * 48, bv, &st_full[s]);
        }
      }
      if (!ok && !*abort_s) fail();
      // Drain: the last copy into every stage has landed before the CTA exits.
      for (int k = 1; k <= kStages && j - k >= 0; ++k) {
        const int jj = j - k;
        mbar_wait(&st_full[jj % kStages], (jj / kStages) & 1);
      }
    }
  } else if (warp == 1 || warp == 14) {
    // ------------------------------------------ MMA issuers (one thread each)
    // warp 1 issues the score MMAs, warp 14 the PV MMAs, so the issue
    // latencies of the two chains overlap.
    if (lane == 0) {
      const uint32_t id_mse = idesc_i8(true, false), id_sgn = idesc_i8(false, false), id_v = idesc_i8(true, true);
      const uint64_t p_desc0 = desc_k_sw128(smem_u32(sm + Sm::kOffP));
      const uint64_t b_desc0 = desc_k_sw128(smem_u32(sm + Sm::kOffB));
      const uint64_t vh_desc0 = desc_k_sw128(smem_u32(sm + Sm::kOffVh));
      int j = 0, s_k = 0;
      bool ok = true;
      for (int item = blockIdx.x; ok && item < A.n_items; item += gridDim.x, ++s_k) {
        int64_t tb, te;
        const int nt_tiles = item_tiles(item, tb, te);
        for (int tj = 0; tj < nt_tiles; ++tj, ++j) {
          const int b = j & 1;
          const uint32_t ph = (j >> 1) & 1;
          if (*abort_s) { ok = false; break; }
          if (warp == 1) {
            const int ib = s_k & 1;
            if (!mbar_wait(&b_full[ib], (s_k >> 1) & 1) || !mbar_wait(&a_full[b], ph) ||
                !mbar_wait(&ds_free[b], ph ^ 1)) { ok = false; break; }
            tc_fence_after();
            const uint32_t d = tmem + kColDs + b * 32;
            const uint32_t a0 = tmem + kColA + b * 128;
            // a1, a2, a3 against B1, B2, B3 (limb-shifted q) into the MSE
            // columns, the sign chunk into its own columns.
            const uint64_t bs = b_desc0 + (((ib * 4 + 3) * 2048) >> 4);
#pragma unroll
            for (int step = 0; step < 12; ++step) {
              const int ch = step >> 2, k = step & 3;
              const uint64_t bq = b_desc0 + (((ib * 4 + ch) * 2048) >> 4);
              umma_i8_ts(d, a0 + ch * 32 + k * 8, bq + ((k * 32) >> 4), id_mse, step != 0);
              if (step < 4) umma_i8_ts(d + 16, a0 + 96 + k * 8, bs + ((k * 32) >> 4), id_sgn, k != 0);
            }
            umma_commit(&s_full[b]);
          } else {
            if (!mbar_wait(&vh_full[b], ph) || !mbar_wait(&p_full[b], ph) || !mbar_wait(&do_free[b], ph ^ 1)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t d = tmem + kColDo + b * 32;
            const uint64_t pb = p_desc0 + ((b * 2048) >> 4);
#pragma unroll
            for (int k = 0; k < 4; ++k) {             // 32 tokens per step = 4 atoms of 8 tokens
#pragma unroll
              for (int limb = 0; limb < 2; ++limb) {  // the two limb chains alternate
                const uint64_t ad = vh_desc0 + ((b * Sm::kVhBytes + limb * kTT * 128 + k * 4096) >> 4);
                umma_i8_ss(d + limb * 16, ad, pb + ((k * 32) >> 4), id_v, k != 0);
              }
            }
            umma_commit(&pv_full[b]);
          }
        }
      }
      if (!ok && !*abort_s) fail();
      // Every MMA this thread issued completes before TMEM is released.
      umma_commit(&drain[warp == 1 ? 0 : 1]);
      mbar_wait(&drain[warp == 1 ? 0 : 1], 0);
    }
  } else if (warp < 6) {
    // ------------------------------------------------- key operands (TMEM)
    const int q = warp & 3;                       // lane quadrant (warps 2..5 -> 2,3,0,1)
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(q * 32) << 16);
    const int row = q * 32 + lane;                // token = TMEM lane this thread writes
    uint32_t k1[4], k2[4], k3[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      k1[u] = tab[u];
      k2[u] = tab[4 + u];
      k3[u] = tab[8 + u];
    }
    int j = 0;
    bool stop = false;
    for (int item = blockIdx.x; !stop && item < A.n_items; item += gridDim.x) {
      int64_t tb, te;
      const int nt_tiles = item_tiles(item, tb, te);
      for (int tj = 0; tj < nt_tiles; ++tj, ++j) {
        const int s = j % kStages;
        const int b = j & 1;
        if (!__all_sync(0xffffffffu, mbar_wait(&st_full[s], (j / kStages) & 1))) {
          if (lane == 0) fail();
          stop = true;
          break;
        }
        const unsigned char* st = sm + s * Sm::kStageStride;
        uint32_t w[kRbk / 4 + 1];
#pragma unroll
        for (int u = 0; u < kRbk / 16; ++u) {
          const uint4 x = reinterpret_cast<const uint4*>(st + row * kRbk)[u];
          w[4 * u] = x.x; w[4 * u + 1] = x.y; w[4 * u + 2] = x.z; w[4 * u + 3] = x.w;
        }
        w[kRbk / 4] = 0u;
        const uint4 sg = reinterpret_cast<const uint4*>(st + kTT * kRbk + row * 16)[0];
        __syncwarp();
        if (lane == 0) mbar_arrive(&st_empty[s]);
        if (!__all_sync(0xffffffffu, mbar_wait(&a_free[b], ((j >> 1) & 1) ^ 1))) {
          if (lane == 0) fail();
          stop = true;
          break;
        }
        tc_fence_after();
        const uint32_t acol = lane_addr + kColA + b * 128;
        // 32 coordinates per iteration (KB words of codes, w[0..KB-1]; the
        // words shift down after each one): nibble selectors, then the three
        // limbs of each coordinate by byte permutes into 8 TMEM columns per limb.
#pragma unroll 1
        for (int qq = 0; qq < 4; ++qq) {
          uint32_t xq[KB + 1];
#pragma unroll
          for (int u = 0; u < KB; ++u) xq[u] = w[u];
          xq[KB] = 0u;
          uint32_t nib[4];
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            const int off = KB * g;               // byte offset of the group
            const int wi = off >> 2, shf = 8 * (off & 3);
            const uint32_t x = shf == 0 ? xq[wi] : __funnelshift_r(xq[wi], xq[wi + 1], shf);
            if (KB == 3) nib[g] = nibbles3(x);
            else if (KB == 2) nib[g] = nibbles2(x);
            else nib[g] = x;                      // 4-bit codes are nibbles already
          }
#pragma unroll
          for (int limb = 0; limb < 3; ++limb) {
            const uint32_t(&t)[4] = limb == 0 ? k1 : (limb == 1 ? k2 : k3);
            uint32_t v8[8];
#pragma unroll
            for (int g = 0; g < 4; ++g) {
              if (KB <= 3) {
                v8[2 * g] = prmt(t[0], t[1], nib[g]);
                v8[2 * g + 1] = prmt(t[0], t[1], nib[g] >> 16);
              } else {
                v8[2 * g] = lut16(t, nib[g] & 0xFFFFu);
                v8[2 * g + 1] = lut16(t, nib[g] >> 16);
              }
            }
            tmem_st8(acol + limb * 32 + qq * 8, v8);
          }
#pragma unroll
          for (int u = 0; u + KB < kRbk / 4 + 1; ++u) w[u] = w[u + KB];
        }
        uint32_t v[32];
        // Sign chunk: column 4 m + u = sign word u AND (0x01010101 << m).
        const uint32_t sw[4] = {sg.x, sg.y, sg.z, sg.w};
#pragma unroll
        for (int m = 0; m < 8; ++m)
#pragma unroll
          for (int u = 0; u < 4; ++u) v[4 * m + u] = sw[u] & (0x01010101u << m);
        tmem_st32(acol + 96, v);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&a_full[b]);
      }
    }
  } else if (warp < 10) {
    // ------------------------------- value operands (smem), value epilogue
    const int row = tid - 192;                    // token within the tile (operands)
    const int q = warp & 3;                       // lane quadrant (warps 6..9 -> 2,3,0,1)
    const int crd = q * 32 + lane;                // coordinate = TMEM lane (epilogue)
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(q * 32) << 16);
    const uint32_t v1t[2] = {tab[12], tab[13]}, v2t[2] = {tab[16], tab[17]};
    int j = 0;
    bool stop = false;
    float acc[2][kRowsTc];                        // even / odd tiles of the item
    // Value epilogue of tile jj (this thread = coordinate crd): wait for its
    // PV product, then for ring slot jj % 4 to carry tag jj (the softmax warps
    // write the tile's corrections and scale, fence, then the tag; the slot is
    // rewritten only after PV(jj + 2), which needs this epilogue's do_free).
    auto value_epilogue = [&](int jj) -> bool {
      const int b2 = jj & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&pv_full[b2], (jj >> 1) & 1))) return false;
      tc_fence_after();
      uint32_t d[32];
      tmem_ld32(lane_addr + kColDo + b2 * 32, d);
      volatile int* tag = reinterpret_cast<volatile int*>(ring + (jj & 3) * 8 + 5);
      bool tag_ok = *tag == jj;
      if (!tag_ok) {
        const uint64_t t0 = globaltimer_ns();
        while (!(tag_ok = (*tag == jj)) && globaltimer_ns() - t0 < 2000000000ull) {
        }
      }
      __threadfence_block();
      const float4 c4 = reinterpret_cast<const float4*>(ring + (jj & 3) * 8)[0];
      const float spv = ring[(jj & 3) * 8 + 4] * v_scale;
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&do_free[b2]);
      if (!__all_sync(0xffffffffu, tag_ok)) return false;
      const float corr[kRowsTc] = {c4.x, c4.y, c4.z, c4.w};
#pragma unroll
      for (int r = 0; r < kRowsTc; ++r) {
        // column (r, weight limb l) = 3 r + l in each value-limb chain
        const float hi = limb_sum3(d + 3 * r), lo = limb_sum3(d + 16 + 3 * r);
        acc[b2][r] = fmaf(acc[b2][r], corr[r], spv * fmaf(lo, 1.f / 128.f, hi));
      }
      return true;
    };
    for (int item = blockIdx.x; !stop && item < A.n_items; item += gridDim.x) {
      int64_t tb, te;
      const int nt_tiles = item_tiles(item, tb, te);
#pragma unroll
      for (int r = 0; r < kRowsTc; ++r) acc[0][r] = acc[1][r] = 0.f;
      for (int tj = 0; tj < nt_tiles; ++tj, ++j) {
        const int s = j % kStages;
        const int b = j & 1;
        if (!__all_sync(0xffffffffu, mbar_wait(&st_full[s], (j / kStages) & 1))) {
          if (lane == 0) fail();
          stop = true;
          break;
        }
        const unsigned char* st = sm + s * Sm::kStageStride;
        uint32_t w[13];
#pragma unroll
        for (int u = 0; u < 3; ++u) {
          const uint4 x = reinterpret_cast<const uint4*>(st + kTT * (kRbk + 16) + row * 48)[u];
          w[4 * u] = x.x; w[4 * u + 1] = x.y; w[4 * u + 2] = x.z; w[4 * u + 3] = x.w;
        }
        w[12] = 0u;
        __syncwarp();
        if (lane == 0) mbar_arrive(&st_empty[s]);
        if (!__all_sync(0xffffffffu, mbar_wait(&vh_free[b], ((j >> 1) & 1) ^ 1))) {
          if (lane == 0) fail();
          stop = true;
          break;
        }
        unsigned char* vh = sm + Sm::kOffVh + b * Sm::kVhBytes;
        // Row `row` (token) of each limb tile: 128 coordinate bytes, M-major,
        // 8-token atoms of 1024 bytes. 32 coordinates (12 code bytes, w[0..2])
        // per iteration; the words shift down after each one.
        const int atom = row >> 3, r8 = row & 7;
#pragma unroll 1
        for (int c2 = 0; c2 < 4; ++c2) {
          const uint32_t x4[4] = {w[0], w[1], w[2], 0u};
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) {          // 16 coordinates = 6 bytes of codes
            uint32_t o1[4], o2[4];
#pragma unroll
            for (int h = 0; h < 2; ++h) {           // 8 codes per half
              const int g = 2 * cc + h;
              const int off = 3 * g, wi = off >> 2, shf = 8 * (off & 3);
              const uint32_t x = shf == 0 ? x4[wi] : __funnelshift_r(x4[wi], x4[wi + 1], shf);
              const uint32_t nb = nibbles3(x);
              o1[2 * h] = prmt(v1t[0], v1t[1], nb);
              o1[2 * h + 1] = prmt(v1t[0], v1t[1], nb >> 16);
              o2[2 * h] = prmt(v2t[0], v2t[1], nb);
              o2[2 * h + 1] = prmt(v2t[0], v2t[1], nb >> 16);
            }
            const int c16 = 2 * c2 + cc;
            const uint32_t off = atom * 1024 + r8 * 128 + ((c16 ^ r8) << 4);
            *reinterpret_cast<uint4*>(vh + off) = make_uint4(o1[0], o1[1], o1[2], o1[3]);
            *reinterpret_cast<uint4*>(vh + kTT * 128 + off) = make_uint4(o2[0], o2[1], o2[2], o2[3]);
          }
#pragma unroll
          for (int u = 0; u < 9; ++u) w[u] = w[u + 3];
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&vh_full[b]);
        // Fold the previous tile of this item (its PV product is under way or done).
        if (tj >= 1 && !value_epilogue(j - 1)) {
          if (lane == 0) fail();
          stop = true;
          break;
        }
      }
      if (stop) break;
      if (!value_epilogue(j - 1)) {
        if (lane == 0) fail();
        break;
      }
      // Rotated-value partials of the item's even and odd tiles (records
      // 2 split + parity; m and l come from the softmax warps).
      const int64_t unit = item / sh.n_splits;
      const int split = item % sh.n_splits;
      const int kv = static_cast<int>(unit % sh.hkv), bb = static_cast<int>(unit / sh.hkv);
      const int G = sh.hq / sh.hkv;
#pragma unroll
      for (int r = 0; r < kRowsTc; ++r) {
        const int64_t qr = (int64_t(bb) * sh.hq + kv * G + r / sh.nq) * sh.nq + r % sh.nq;
        float* pr = a.part + (qr * sh.n_parts + 2 * split) * (kD + 2) + crd;
        pr[0] = acc[0][r];
        pr[kD + 2] = acc[1][r];
      }
    }
  } else if (warp < 14) {
    // ------------------- scores and softmax: even and odd tiles kept apart
    constexpr int wg = 0;
    const int cw = warp - 10;                     // warp within the group
    const int q = warp & 3;                       // lane quadrant (2,3,0,1 per group)
    const int lrow = q * 32 + lane;               // TMEM lane = token
    const int bar_id = 1 + wg;
    float* gred = red + wg * 64;
    float* gred2 = red2 + wg * 16;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(q * 32) << 16);
    const float alpha = static_cast<float>(dev::kSqrtHalfPi / kD);
    constexpr float kLog2e = 1.4426950408889634f;
    constexpr float kMagic = 12582912.f;          // 1.5 * 2^23: x + kMagic rounds x to an integer
    // Byte offsets of this token's column in the 12 used rows of a weight tile.
    uint32_t poff[12];
#pragma unroll
    for (int n = 0; n < 12; ++n) poff[n] = sw_byte(n, lrow);
    int j = 0, item_idx = 0;
    bool stop = false;
    for (int item = blockIdx.x; item < A.n_items && !stop; item += gridDim.x, ++item_idx) {
      int64_t tb, te;
      const int nt_tiles = item_tiles(item, tb, te);
      const int64_t unit = item / sh.n_splits;
      const int split = item % sh.n_splits;
      const int kv = static_cast<int>(unit % sh.hkv), bb = static_cast<int>(unit / sh.hkv);
      const int G = sh.hq / sh.hkv;
      const int64_t row0 = item_row0(item);
      int64_t qrow[kRowsTc];
#pragma unroll
      for (int r = 0; r < kRowsTc; ++r)
        qrow[r] = (int64_t(bb) * sh.hq + kv * G + r / sh.nq) * sh.nq + r % sh.nq;
      // ---- item prologue: row scales, the item's largest ||v||; group 0
      // also writes the item's B tiles.
      const int ib = item_idx & 1;
      float sq[kRowsTc], ss[kRowsTc], ssum[kRowsTc], sp;
      {
        const int crd = lrow;                     // thread = coordinate here
        const float jscale = __uint_as_float(static_cast<uint32_t>(127 - (crd & 7)) << 23);   // 2^-(i mod 8)
        float qv[kRowsTc], sv[kRowsTc], loc[13];
#pragma unroll
        for (int r = 0; r < kRowsTc; ++r) {
          qv[r] = a.qs[qrow[r] * 2 * kD + crd];
          sv[r] = a.qs[qrow[r] * 2 * kD + kD + crd];
          loc[r] = fabsf(qv[r]);
          loc[4 + r] = fabsf(sv[r]) * jscale;
          loc[8 + r] = sv[r];
        }
        float vm = 0.f;
        for (int64_t t = tb + lrow; t < te; t += kTT) vm = fmaxf(vm, __ldg(a.vnorm + row0 + t));
        loc[12] = vm;
#pragma unroll
        for (int u = 0; u < 13; ++u) {
          const float x = (u >= 8 && u < 12) ? warp_sum(loc[u]) : warp_max(loc[u]);
          if (lane == 0) gred[cw * 16 + u] = x;
        }
        wg_sync(bar_id);
        float tot[13];
#pragma unroll
        for (int u = 0; u < 13; ++u) {
          float x = gred[u];
#pragma unroll
          for (int w2 = 1; w2 < 4; ++w2) x = (u >= 8 && u < 12) ? x + gred[w2 * 16 + u] : fmaxf(x, gred[w2 * 16 + u]);
          tot[u] = x;
        }
#pragma unroll
        for (int r = 0; r < kRowsTc; ++r) {
          sq[r] = tot[r] > 0.f ? tot[r] / 127.f : 1.f;
          ss[r] = tot[4 + r] > 0.f ? tot[4 + r] / 127.f : 1.f;
          ssum[r] = tot[8 + r];
        }
        // Weights p ||v|| <= max ||v|| of the item (p <= 1): three int8 limbs.
        sp = tot[12] > 0.f ? tot[12] / 127.f : 1.f;
        if (wg == 0) {
          // B tiles: B1/B2/B3 rows 4 r + w hold limb w, w-1, w-2 of q_rot row r;
          // Bs rows 4 r + l hold limb l of s' at K position 16 (i mod 8) + i / 8.
          unsigned char* bt = sm + Sm::kOffB + ib * 4 * 2048;
          const int ks = 16 * (crd & 7) + (crd >> 3);
#pragma unroll
          for (int r = 0; r < kRowsTc; ++r) {
            int lq[4], ls[4];
            limbs4(qv[r] / sq[r], lq);
            limbs4(sv[r] * jscale / ss[r], ls);
#pragma unroll
            for (int w2 = 0; w2 < 4; ++w2) {
              bt[sw_byte(4 * r + w2, crd)] = static_cast<unsigned char>(static_cast<int8_t>(lq[w2]));
              bt[2048 + sw_byte(4 * r + w2, crd)] =
                  static_cast<unsigned char>(static_cast<int8_t>(w2 >= 1 ? lq[w2 - 1] : 0));
              bt[4096 + sw_byte(4 * r + w2, crd)] =
                  static_cast<unsigned char>(static_cast<int8_t>(w2 >= 2 ? lq[w2 - 2] : 0));
              bt[6144 + sw_byte(4 * r + w2, ks)] = static_cast<unsigned char>(static_cast<int8_t>(ls[w2]));
            }
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&b_full[ib]);
        }
      }
      const float inv_sp = 1.f / sp;
      float kq[kRowsTc], ks2[kRowsTc];
      const float kr = a.scale * alpha;
#pragma unroll
      for (int r = 0; r < kRowsTc; ++r) {
        kq[r] = a.scale * k_scale * sq[r];
        ks2[r] = 2.f * ss[r];
      }
      // Running maximum and sum of the item's even and odd tiles, kept apart:
      // the value warps accumulate the two parities separately and each
      // leaves its own partial record.
      // m_run / l_part: state of the parity of the tile being processed;
      // m_oth / l_oth: the other parity's (swapped after every tile).
      float m_run[kRowsTc], l_part[kRowsTc], m_oth[kRowsTc], l_oth[kRowsTc];
#pragma unroll
      for (int r = 0; r < kRowsTc; ++r) {
        m_run[r] = m_oth[r] = -INFINITY;
        l_part[r] = l_oth[r] = 0.f;
      }
      const int j0 = j;
      // Norms are loaded one tile ahead.
      float kn_n = 0.f, rn_n = 0.f, vn_n = 0.f;
      if (lrow < te - tb) {
        kn_n = __ldg(a.knorm + row0 + tb + lrow);
        rn_n = __ldg(a.krnorm + row0 + tb + lrow);
        vn_n = __ldg(a.vnorm + row0 + tb + lrow);
      }
      for (int tj = 0; tj < nt_tiles; ++tj) {
        const int jt = j0 + tj;
        const int b = jt & 1;
        const int64_t t0 = tb + int64_t(tj) * kTT;
        const int nt = static_cast<int>((te - t0 < kTT) ? te - t0 : kTT);
        const bool valid = lrow < nt;
        const float kn = kn_n, rn = rn_n, vn = vn_n;
        if (t0 + kTT + lrow < te) {
          kn_n = __ldg(a.knorm + row0 + t0 + kTT + lrow);
          rn_n = __ldg(a.krnorm + row0 + t0 + kTT + lrow);
          vn_n = __ldg(a.vnorm + row0 + t0 + kTT + lrow);
        }
        const bool ok = __all_sync(0xffffffffu, mbar_wait(&s_full[b], (jt >> 1) & 1));
        tc_fence_after();
        uint32_t d[32];
        tmem_ld32(lane_addr + kColDs + b * 32, d);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ds_free[b]);
        float score[kRowsTc];
        bool need = false;
#pragma unroll
        for (int r = 0; r < kRowsTc; ++r) {
          // weights 0, 1, 2 of the key limb products (weight 3 is below 1e-6)
          const float mse = limb_sum3(d + 4 * r);
          const float sgn = limb_sum4(d + 16 + 4 * r);
          const float qjl = fmaf(ks2[r], sgn, -ssum[r]);
          score[r] = valid ? fmaf(kq[r] * kn, mse, kr * rn * qjl) : -INFINITY;
          need |= score[r] > m_run[r];
        }
        if (a.scores_out && valid) {
#pragma unroll
          for (int r = 0; r < kRowsTc; ++r) a.scores_out[qrow[r] * sh.n_ctx + t0 + lrow] = score[r];
        }
        float corr[kRowsTc];
#pragma unroll
        for (int r = 0; r < kRowsTc; ++r) corr[r] = 1.f;
        // The running maximum moves only when some score of the tile exceeds it.
        if (wg_sync_or(bar_id, need || !ok || *abort_s != 0)) {
          if (wg_sync_or(bar_id, !ok || *abort_s != 0)) {
            if (!ok && lane == 0 && cw == 0) fail();
            stop = true;
            break;
          }
#pragma unroll
          for (int r = 0; r < kRowsTc; ++r) {
            const float mx = warp_max(score[r]);
            if (lane == 0) gred[cw * 16 + r] = mx;
          }
          wg_sync(bar_id);
#pragma unroll
          for (int r = 0; r < kRowsTc; ++r) {
            float mx = gred[r];
#pragma unroll
            for (int w2 = 1; w2 < 4; ++w2) mx = fmaxf(mx, gred[w2 * 16 + r]);
            const float m_new = fmaxf(m_run[r], mx);
            corr[r] = (m_run[r] == -INFINITY) ? 0.f : ex2((m_run[r] - m_new) * kLog2e);
            l_part[r] *= corr[r];
            m_run[r] = m_new;
          }
        }
        float p[kRowsTc];
#pragma unroll
        for (int r = 0; r < kRowsTc; ++r) {
          p[r] = valid ? ex2((score[r] - m_run[r]) * kLog2e) : 0.f;
          l_part[r] += p[r];
        }
        // Weight limbs into the P tile (row 3 r + limb, column = token); the
        // tile's corrections and scale go to ring[jt % 4] for the value warps.
        if (!__all_sync(0xffffffffu, mbar_wait(&p_free[b], ((jt >> 1) & 1) ^ 1)) && lane == 0) fail();
        if (lrow == 0) {
          float* slot = ring + (jt & 3) * 8;
          reinterpret_cast<float4*>(slot)[0] = make_float4(corr[0], corr[1], corr[2], corr[3]);
          slot[4] = sp;
          __threadfence_block();
          *reinterpret_cast<volatile int*>(slot + 5) = jt;
        }
        unsigned char* pt = sm + Sm::kOffP + b * 2048;
        const float wv = vn * inv_sp;
#pragma unroll
        for (int r = 0; r < kRowsTc; ++r) {
          // X = rint(x 2^14) < 2^21 in the low mantissa bits; its base-128
          // digits are the limbs: x ~ d1 + d2/128 + d3/128^2.
          const float x = fminf(p[r] * wv, 127.f);
          const uint32_t X = __float_as_uint(fmaf(x, 16384.f, kMagic)) - 0x4B400000u;
          pt[poff[3 * r]] = static_cast<unsigned char>(X >> 14);
          pt[poff[3 * r + 1]] = static_cast<unsigned char>((X >> 7) & 127u);
          pt[poff[3 * r + 2]] = static_cast<unsigned char>(X & 127u);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[b]);
#pragma unroll
        for (int r = 0; r < kRowsTc; ++r) {
          const float tm = m_run[r], tl = l_part[r];
          m_run[r] = m_oth[r];
          l_part[r] = l_oth[r];
          m_oth[r] = tm;
          l_oth[r] = tl;
        }
      }
      j = j0 + nt_tiles;
      if (stop) break;
      // Softmax statistics of the two partials (the value warps write acc).
      // m_run / l_part now hold the parity of tile j0 + nt_tiles, m_oth / l_oth
      // the other one.
      const int par_run = (j0 + nt_tiles) & 1;
#pragma unroll
      for (int par = 0; par < 2; ++par) {
        const bool use_run = par == par_run;
        float lsum[kRowsTc];
#pragma unroll
        for (int r = 0; r < kRowsTc; ++r) {
          const float x = warp_sum(use_run ? l_part[r] : l_oth[r]);
          if (lane == 0) gred2[cw * 4 + r] = x;
        }
        wg_sync(bar_id);
#pragma unroll
        for (int r = 0; r < kRowsTc; ++r) lsum[r] = gred2[r] + gred2[4 + r] + gred2[8 + r] + gred2[12 + r];
        wg_sync(bar_id);
        if (lrow == 0) {
          // record 2 split + parity of the tiles' index j
          const int rec = 2 * split + par;
#pragma unroll
          for (int r = 0; r < kRowsTc; ++r) {
            float* pr = a.part + (qrow[r] * sh.n_parts + rec) * (kD + 2);
            pr[kD] = use_run ? m_run[r] : m_oth[r];
            pr[kD + 1] = lsum[r];
          }
        }
      }
    }
  }

  // ------------------------------------------------------------- teardown
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    __syncwarp();
    tmem_dealloc(tmem, kTmemColsTc);
  }
}

}  // namespace

bool tc_decode_supported(const DecodeArgs& v) {
  const DecodeShape& s = v.sh;
  if (s.d != kD || s.vbits != 3 || s.rows_per_cta != kRowsTc || s.row_blocks != 1) return false;
  if (s.kbits < 2 || s.kbits > 4) return false;
  // Bulk copies need 16-byte aligned sources: plane bases and stream offsets.
  if (!aligned(v.kidx, 16) || !aligned(v.ksign, 16) || !aligned(v.vidx, 16)) return false;
  return true;
}

cudaError_t tc_decode_launch(const DecodeArgs& v, cudaStream_t st) {
  TcDecodeArgs A{};
  A.v = v;
  A.n_items = static_cast<int>(int64_t(v.sh.batch) * v.sh.hkv * v.sh.n_splits);
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = A.n_items < sms ? A.n_items : sms;
  cudaError_t e;
  switch (v.sh.kbits) {
    case 2:
      e = cudaFuncSetAttribute(decode_tc_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, TcSm<2>::kBytes);
      if (e == cudaSuccess) decode_tc_kernel<2><<<grid, kThreadsTc, TcSm<2>::kBytes, st>>>(A);
      break;
    case 3:
      e = cudaFuncSetAttribute(decode_tc_kernel<3>, cudaFuncAttributeMaxDynamicSharedMemorySize, TcSm<3>::kBytes);
      if (e == cudaSuccess) decode_tc_kernel<3><<<grid, kThreadsTc, TcSm<3>::kBytes, st>>>(A);
      break;
    default:
      e = cudaFuncSetAttribute(decode_tc_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, TcSm<4>::kBytes);
      if (e == cudaSuccess) decode_tc_kernel<4><<<grid, kThreadsTc, TcSm<4>::kBytes, st>>>(A);
      break;
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace tq
