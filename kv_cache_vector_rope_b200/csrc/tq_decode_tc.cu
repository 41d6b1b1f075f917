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
//   scores  S[t][r] = sum_i c_K[code_ti] q_r,i  and  sum_i bit_ti s_r,i.
//           A (TMEM, one lane per token): the key codebook value of every
//           coordinate as three int8 limbs (c = sc (a1 + a2/128 + a3/128^2))
//           and the sign bits as 0/1 bytes. B (smem): q_rot and s = S q_rot
//           of the four rows as three int8 limbs each. int32 accumulation is
//           exact. Three codebook limbs are needed because a codebook error
//           repeats on every coordinate holding that code: with two limbs the
//           2-bit codebook alone moves scores by ~1e-4 of |q||k|/d.
//   values  O[i][r] = sum_t c_V[code_ti] w_r,t with w = p ||v||.
//           A (smem, M-major): the value codebook value as two int8 limbs
//           per coordinate, one 128-byte row per token. B (smem): the tile's
//           weights as two int8 limbs per row with a per-tile scale. Each
//           tile's int32 result is folded into fp32 accumulators (one
//           coordinate per thread) with the online-softmax correction.
// Roles (448 threads, one persistent CTA per SM):
//   warp 0   bulk copies of the packed index / sign planes into a 3-stage ring
//   warp 1   TMEM owner and single-thread tcgen05.mma issuer
//   WG A     key dequantisation into TMEM          (thread = token)
//   WG B     value dequantisation into smem        (thread = token)
//   WG C     score epilogue, online softmax, weight limbs (thread = token)
//            and the value epilogue                (thread = coordinate)
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
constexpr int kThreadsTc = 448;        // 14 warps
constexpr int kRowsTc = 4;

// TMEM columns (32-bit): A_score [0,128): a1 | a2 | a3 | sign bytes (32 each);
// D_score x2 at 128, 192 (64 each: four 16-column chains); D_o x2 at 256, 288.
constexpr uint32_t kColA = 0, kColDs = 128, kColDo = 256, kTmemColsTc = 512;
constexpr uint32_t kDsCols = 64;

// Instruction descriptor, kind::i8: s32 D, signed A/B, M = 128, N = 16.
__host__ __device__ constexpr uint32_t idesc_i8(bool a_mn_major) {
  return (2u << 4) | (1u << 7) | (1u << 10) | ((a_mn_major ? 1u : 0u) << 15) | ((16u >> 3) << 17) |
         ((128u >> 4) << 24);
}

template <int KB>
struct TcSm {
  static constexpr int kRbk = kD * KB / 8;
  static constexpr int kStageBytes = kTT * (kRbk + 16 + 48);       // kidx | ksign | vidx
  static constexpr int kOffStage = 0;
  static constexpr int kOffVh = 3 * ((kStageBytes + 1023) / 1024) * 1024;   // 1024-aligned
  static constexpr int kVhBytes = 2 * kTT * 128;                    // two limbs x 128 tokens x 128 B
  static constexpr int kOffP = kOffVh + 2 * kVhBytes;               // 2 x [16 rows x 128 B]
  static constexpr int kOffB = kOffP + 2 * 2048;                    // 2 items x (Q limbs | S limbs)
  static constexpr int kOffBar = kOffB + 2 * 4096;
  static constexpr int kNumBars = 2 * kStages + 2 + 2 * 2 * 6 + 2 + 1;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  // misc: tmem base, abort | item scales [2][16] | ring [2][8] | scratch [16] |
  // reductions [4 warps][8] | codebook limb tables (ka1 ka2 ka3 va1 va2, 4 words each) | scales (key, value)
  static constexpr int kOffScale = kOffMisc + 16;
  static constexpr int kOffRing = kOffScale + 2 * 16 * 4;
  static constexpr int kOffScr = kOffRing + 2 * 8 * 4;
  static constexpr int kOffRed = kOffScr + 16 * 4;
  static constexpr int kOffTab = kOffRed + 4 * 8 * 4;
  static constexpr int kBytes = kOffTab + 32 * 4 + 1024;
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

// 8 three-bit codes (24 bits) -> two PRMT selectors of four nibbles each.
__device__ __forceinline__ void spread3(uint32_t x, uint32_t& lo, uint32_t& hi) {
  const uint32_t y = (x & 0xFFFu) | ((x << 4) & 0x0FFF0000u);
  const uint32_t z = (y & 0x00070007u) | ((y << 1) & 0x00700070u) | ((y << 2) & 0x07000700u) | ((y << 3) & 0x70007000u);
  lo = z & 0xFFFFu;
  hi = z >> 16;
}
// 8 two-bit codes (16 bits) -> nibble selectors.
__device__ __forceinline__ void spread2(uint32_t x, uint32_t& lo, uint32_t& hi) {
  const uint32_t y = (x & 0xFFu) | ((x << 8) & 0x00FF0000u);
  const uint32_t z = (y & 0x00030003u) | ((y << 2) & 0x00300030u) | ((y << 4) & 0x03000300u) | ((y << 6) & 0x30003000u);
  lo = z & 0xFFFFu;
  hi = z >> 16;
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
// Four sign bits -> four 0/1 bytes.
__device__ __forceinline__ uint32_t bits4_to_bytes(uint32_t n4) { return (n4 * 0x00204081u) & 0x01010101u; }

__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&v)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(v[0]),
               "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
               : "memory");
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
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
// Three int8 limbs of x / scale (|x / scale| <= 127): x ~ scale (l0 + l1/128 + l2/16384).
__device__ __forceinline__ void limbs3(float x, float inv_scale, int& l0, int& l1, int& l2) {
  const float r0 = x * inv_scale;
  l0 = __float2int_rn(r0);
  const float r1 = (r0 - static_cast<float>(l0)) * 128.f;
  l1 = __float2int_rn(r1);
  l2 = __float2int_rn((r1 - static_cast<float>(l1)) * 128.f);
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
  uint64_t* a_full = bars + 2 * kStages;          // [1]
  uint64_t* a_free = a_full + 1;                  // [1]
  uint64_t* s_full = a_free + 1;                  // [2]
  uint64_t* ds_free = s_full + 2;                 // [2]
  uint64_t* vh_full = ds_free + 2;                // [2]
  uint64_t* vh_free = vh_full + 2;                // [2]
  uint64_t* p_full = vh_free + 2;                 // [2]
  uint64_t* p_free = p_full + 2;                  // [2]
  uint64_t* pv_full = p_free + 2;                 // [2]
  uint64_t* do_free = pv_full + 2;                // [2]
  uint64_t* b_full = do_free + 2;                 // [2] per item parity
  uint64_t* drain = b_full + 2;                   // [1]
  uint32_t* tmem_base_s = reinterpret_cast<uint32_t*>(sm + Sm::kOffMisc);
  volatile int* abort_s = reinterpret_cast<volatile int*>(sm + Sm::kOffMisc + 4);
  float* item_scale = reinterpret_cast<float*>(sm + Sm::kOffScale);   // [2][16]: sq[4], ss[4], ssum[4]
  float* ring = reinterpret_cast<float*>(sm + Sm::kOffRing);          // [2][8]: corr[4], sp[4]
  float* red = reinterpret_cast<float*>(sm + Sm::kOffRed);            // [4 warps][8]
  float* scr = reinterpret_cast<float*>(sm + Sm::kOffScr);            // [16]
  uint32_t* tab = reinterpret_cast<uint32_t*>(sm + Sm::kOffTab);      // ka1 ka2 ka3 va1 va2 (4 words each)
  float* cb_scale = reinterpret_cast<float*>(sm + Sm::kOffTab + 20 * 4);   // key, value codebook scales

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const DecodeShape& sh = a.sh;

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&st_full[s], 1);
      mbar_init(&st_empty[s], 8);
    }
    mbar_init(a_full, 4);
    mbar_init(a_free, 1);
    for (int b = 0; b < 2; ++b) {
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
    mbar_init(drain, 1);
    *abort_s = 0;
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
          unsigned char* st = sm + Sm::kOffStage + s * ((Sm::kStageBytes + 1023) / 1024) * 1024;
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
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t id_s = idesc_i8(false), id_v = idesc_i8(true);
      const uint64_t p_desc0 = desc_k_sw128(smem_u32(sm + Sm::kOffP));
      const uint64_t b_desc0 = desc_k_sw128(smem_u32(sm + Sm::kOffB));
      const uint64_t vh_desc0 = desc_k_sw128(smem_u32(sm + Sm::kOffVh));
      int total = 0;
      for (int item = blockIdx.x; item < A.n_items; item += gridDim.x) {
        int64_t tb, te;
        total += item_tiles(item, tb, te);
      }
      int ns = 0, np = 0;                 // next score tile, next PV tile
      int s_item = blockIdx.x, s_k = 0, s_left = 0;
      if (s_item < A.n_items) {
        int64_t tb, te;
        s_left = item_tiles(s_item, tb, te);
      }
      uint64_t last = globaltimer_ns();
      while (np < total) {
        if (*abort_s) break;
        bool progress = false;
        if (ns < total) {
          const int b = ns & 1;
          const int ib = s_k & 1;
          if (mbar_try_wait(&b_full[ib], (s_k >> 1) & 1) && mbar_try_wait(a_full, ns & 1) &&
              mbar_try_wait(&ds_free[b], ((ns >> 1) & 1) ^ 1)) {
            tc_fence_after();
            const uint32_t d = tmem + kColDs + b * kDsCols;
            const uint64_t bq = b_desc0 + ((ib * 4096) >> 4), bsg = b_desc0 + ((ib * 4096 + 2048) >> 4);
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {       // a1, a2, a3 against q limbs; sign bytes against s limbs
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                const uint64_t bd = (ch == 3 ? bsg : bq) + ((k * 32) >> 4);
                umma_i8_ts(d + ch * 16, tmem + kColA + ch * 32 + k * 8, bd, id_s, k != 0);
              }
            }
            umma_commit(&s_full[b]);
            umma_commit(a_free);
            ++ns;
            if (--s_left == 0) {           // next item of this CTA
              s_item += gridDim.x;
              ++s_k;
              if (s_item < A.n_items) {
                int64_t tb, te;
                s_left = item_tiles(s_item, tb, te);
              }
            }
            progress = true;
          }
        }
        if (np < ns) {
          const int b = np & 1;
          const uint32_t ph = (np >> 1) & 1;
          if (mbar_try_wait(&vh_full[b], ph) && mbar_try_wait(&p_full[b], ph) &&
              mbar_try_wait(&do_free[b], ph ^ 1)) {
            tc_fence_after();
            const uint32_t d = tmem + kColDo + b * 32;
            const uint64_t pb = p_desc0 + ((b * 2048) >> 4);
#pragma unroll
            for (int limb = 0; limb < 2; ++limb) {
#pragma unroll
              for (int k = 0; k < 4; ++k) {           // 32 tokens per step = 4 atoms of 8 tokens
                const uint64_t ad = vh_desc0 + ((b * Sm::kVhBytes + limb * kTT * 128 + k * 4096) >> 4);
                umma_i8_ss(d + limb * 16, ad, pb + ((k * 32) >> 4), id_v, k != 0);
              }
            }
            umma_commit(&pv_full[b]);
            umma_commit(&vh_free[b]);
            umma_commit(&p_free[b]);
            ++np;
            progress = true;
          }
        }
        if (progress) {
          last = globaltimer_ns();
        } else if (globaltimer_ns() - last > 2000000000ull) {
          fail();
          break;
        }
      }
    }
  } else if (warp < 6) {
    // ----------------------------------------------- WG A: key dequantisation
    const int t = tid - 64;                       // token within the tile = TMEM lane
    const int q = warp & 3;                       // lane quadrant (warps 2..5 -> 2,3,0,1)
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(q * 32) << 16);
    const int row = q * 32 + lane;                // TMEM lane this thread writes
    uint32_t k1[4], k2[4], k3[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      k1[u] = tab[u];
      k2[u] = tab[4 + u];
      k3[u] = tab[8 + u];
    }
    (void)t;
    int j = 0;
    for (int item = blockIdx.x; item < A.n_items; item += gridDim.x) {
      int64_t tb, te;
      const int nt_tiles = item_tiles(item, tb, te);
      bool stop = false;
      for (int tj = 0; tj < nt_tiles; ++tj, ++j) {
        const int s = j % kStages;
        if (!__all_sync(0xffffffffu, mbar_wait(&st_full[s], (j / kStages) & 1))) {
          if (lane == 0) fail();
          stop = true;
          break;
        }
        const unsigned char* st = sm + Sm::kOffStage + s * ((Sm::kStageBytes + 1023) / 1024) * 1024;
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
        if (!__all_sync(0xffffffffu, mbar_wait(a_free, (j & 1) ^ 1))) {
          if (lane == 0) fail();
          stop = true;
          break;
        }
        tc_fence_after();
        const uint32_t sgw[4] = {sg.x, sg.y, sg.z, sg.w};
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {           // 32 coordinates per chunk
          uint32_t v1[8], v2[8], v3[8], vb[8];
#pragma unroll
          for (int g2 = 0; g2 < 4; ++g2) {          // 8 codes per group
            const int g = ch * 4 + g2;
            const int off = KB * g;                 // byte offset of the group
            const int wi = off >> 2, shf = 8 * (off & 3);
            const uint32_t x = shf == 0 ? w[wi] : __funnelshift_r(w[wi], w[wi + 1], shf);
            uint32_t lo = 0u, hi = 0u;
            if (KB == 3) {
              spread3(x, lo, hi);
            } else if (KB == 2) {
              spread2(x, lo, hi);
            }
            if (KB <= 3) {
              v1[2 * g2] = prmt(k1[0], k1[1], lo);
              v1[2 * g2 + 1] = prmt(k1[0], k1[1], hi);
              v2[2 * g2] = prmt(k2[0], k2[1], lo);
              v2[2 * g2 + 1] = prmt(k2[0], k2[1], hi);
              v3[2 * g2] = prmt(k3[0], k3[1], lo);
              v3[2 * g2 + 1] = prmt(k3[0], k3[1], hi);
            } else {                                // 4-bit codes: nibbles already
              v1[2 * g2] = lut16(k1, x & 0xFFFFu);
              v1[2 * g2 + 1] = lut16(k1, x >> 16);
              v2[2 * g2] = lut16(k2, x & 0xFFFFu);
              v2[2 * g2 + 1] = lut16(k2, x >> 16);
              v3[2 * g2] = lut16(k3, x & 0xFFFFu);
              v3[2 * g2 + 1] = lut16(k3, x >> 16);
            }
          }
#pragma unroll
          for (int n = 0; n < 8; ++n) vb[n] = bits4_to_bytes((sgw[ch] >> (4 * n)) & 15u);
          tmem_st8(lane_addr + kColA + 0 + ch * 8, v1);
          tmem_st8(lane_addr + kColA + 32 + ch * 8, v2);
          tmem_st8(lane_addr + kColA + 64 + ch * 8, v3);
          tmem_st8(lane_addr + kColA + 96 + ch * 8, vb);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(a_full);
      }
      if (stop) break;
    }
  } else if (warp < 10) {
    // --------------------------------------------- WG B: value dequantisation
    const int row = tid - 192;                    // token within the tile
    const uint32_t v1t[2] = {tab[12], tab[13]}, v2t[2] = {tab[16], tab[17]};
    int j = 0;
    for (int item = blockIdx.x; item < A.n_items; item += gridDim.x) {
      int64_t tb, te;
      const int nt_tiles = item_tiles(item, tb, te);
      bool stop = false;
      for (int tj = 0; tj < nt_tiles; ++tj, ++j) {
        const int s = j % kStages;
        const int b = j & 1;
        if (!__all_sync(0xffffffffu, mbar_wait(&st_full[s], (j / kStages) & 1))) {
          if (lane == 0) fail();
          stop = true;
          break;
        }
        const unsigned char* st = sm + Sm::kOffStage + s * ((Sm::kStageBytes + 1023) / 1024) * 1024;
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
        // 8-token atoms of 1024 bytes.
        const int atom = row >> 3, r8 = row & 7;
#pragma unroll
        for (int c16 = 0; c16 < 8; ++c16) {        // 16 coordinates = 6 bytes of codes
          uint32_t o1[4], o2[4];
#pragma unroll
          for (int h = 0; h < 2; ++h) {             // 8 codes per half
            const int g = 2 * c16 + h;
            const int off = 3 * g, wi = off >> 2, shf = 8 * (off & 3);
            const uint32_t x = shf == 0 ? w[wi] : __funnelshift_r(w[wi], w[wi + 1], shf);
            uint32_t lo, hi;
            spread3(x, lo, hi);
            o1[2 * h] = prmt(v1t[0], v1t[1], lo);
            o1[2 * h + 1] = prmt(v1t[0], v1t[1], hi);
            o2[2 * h] = prmt(v2t[0], v2t[1], lo);
            o2[2 * h + 1] = prmt(v2t[0], v2t[1], hi);
          }
          const uint32_t off = atom * 1024 + r8 * 128 + ((c16 ^ r8) << 4);
          *reinterpret_cast<uint4*>(vh + off) = make_uint4(o1[0], o1[1], o1[2], o1[3]);
          *reinterpret_cast<uint4*>(vh + kTT * 128 + off) = make_uint4(o2[0], o2[1], o2[2], o2[3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&vh_full[b]);
      }
      if (stop) break;
    }
  } else {
    // ------------------------------------- WG C: scores, softmax, epilogues
    const int cw = warp - 10;                     // 0..3
    const int q = warp & 3;                       // lane quadrant (warps 10..13 -> 2,3,0,1)
    const int lrow = q * 32 + lane;               // TMEM lane = token / coordinate
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(q * 32) << 16);
    const float alpha = static_cast<float>(dev::kSqrtHalfPi / kD);
    int j = 0, item_idx = 0;
    bool stop = false;
    for (int item = blockIdx.x; item < A.n_items && !stop; item += gridDim.x, ++item_idx) {
      int64_t tb, te;
      const int nt_tiles = item_tiles(item, tb, te);
      const int64_t unit = item / sh.n_splits;
      const int split = item % sh.n_splits;
      const int kv = static_cast<int>(unit % sh.hkv), bb = static_cast<int>(unit / sh.hkv);
      const int G = sh.hq / sh.hkv;
      int64_t qrow[kRowsTc];
#pragma unroll
      for (int r = 0; r < kRowsTc; ++r)
        qrow[r] = (int64_t(bb) * sh.hq + kv * G + r / sh.nq) * sh.nq + r % sh.nq;
      // B operands of this item: rows (r, limb) of q_rot and s as int8, K-major.
      const int ib = item_idx & 1;
      unsigned char* bq = sm + Sm::kOffB + ib * 4096;
      float* isc = item_scale + ib * 16;          // sq[4] | ss[4] | ssum[4]
      {
        // ct = coordinate i: row scales first (max |q_r|, max |s_r| over i).
        float qv[kRowsTc], sv[kRowsTc];
#pragma unroll
        for (int r = 0; r < kRowsTc; ++r) {
          qv[r] = a.qs[qrow[r] * 2 * kD + lrow];
          sv[r] = a.qs[qrow[r] * 2 * kD + kD + lrow];
        }
#pragma unroll
        for (int r = 0; r < kRowsTc; ++r) {
          const float mq = warp_max(fabsf(qv[r])), ms = warp_max(fabsf(sv[r]));
          const float ssum = warp_sum(sv[r]);
          if (lane == 0) {
            red[cw * 8 + r] = mq;
            red[cw * 8 + 4 + r] = ms;
            scr[cw * 4 + r] = ssum;
          }
        }
        wg_sync(2);
        float sq[kRowsTc], ss[kRowsTc];
#pragma unroll
        for (int r = 0; r < kRowsTc; ++r) {
          float mq = 0.f, ms = 0.f, su = 0.f;
#pragma unroll
          for (int w2 = 0; w2 < 4; ++w2) {
            mq = fmaxf(mq, red[w2 * 8 + r]);
            ms = fmaxf(ms, red[w2 * 8 + 4 + r]);
            su += scr[w2 * 4 + r];
          }
          sq[r] = mq > 0.f ? mq / 127.f : 1.f;
          ss[r] = ms > 0.f ? ms / 127.f : 1.f;
          if (lrow == 0) {
            isc[r] = sq[r];
            isc[4 + r] = ss[r];
            isc[8 + r] = su;
          }
        }
        // Write limbs: B row n = 3 r + l holds limb l of row r over coordinates.
#pragma unroll
        for (int r = 0; r < kRowsTc; ++r) {
          int l0, l1, l2;
          limbs3(qv[r], 1.f / sq[r], l0, l1, l2);
          bq[sw_byte(3 * r + 0, lrow)] = static_cast<unsigned char>(static_cast<int8_t>(l0));
          bq[sw_byte(3 * r + 1, lrow)] = static_cast<unsigned char>(static_cast<int8_t>(l1));
          bq[sw_byte(3 * r + 2, lrow)] = static_cast<unsigned char>(static_cast<int8_t>(l2));
          limbs3(sv[r], 1.f / ss[r], l0, l1, l2);
          bq[2048 + sw_byte(3 * r + 0, lrow)] = static_cast<unsigned char>(static_cast<int8_t>(l0));
          bq[2048 + sw_byte(3 * r + 1, lrow)] = static_cast<unsigned char>(static_cast<int8_t>(l1));
          bq[2048 + sw_byte(3 * r + 2, lrow)] = static_cast<unsigned char>(static_cast<int8_t>(l2));
        }
        // Rows 12..15 are zero.
#pragma unroll
        for (int n = 12; n < 16; ++n) {
          bq[sw_byte(n, lrow)] = 0;
          bq[2048 + sw_byte(n, lrow)] = 0;
        }
        fence_proxy_async_smem();
        wg_sync(2);
        __syncwarp();
        if (lane == 0) mbar_arrive(&b_full[ib]);
      }
      float m_run[kRowsTc], l_run[kRowsTc], acc[kRowsTc];
#pragma unroll
      for (int r = 0; r < kRowsTc; ++r) {
        m_run[r] = -INFINITY;
        l_run[r] = 0.f;
        acc[r] = 0.f;
      }
      const int64_t row0 = item_row0(item);
      // Value epilogue of tile jj (this thread = coordinate ct).
      auto value_epilogue = [&](int jj) -> bool {
        const int bb2 = jj & 1;
        if (!__all_sync(0xffffffffu, mbar_wait(&pv_full[bb2], (jj >> 1) & 1))) return false;
        tc_fence_after();
        uint32_t d[32];
        uint32_t d0[16], d1[16];
        tmem_ld16(lane_addr + kColDo + bb2 * 32, d0);
        tmem_ld16(lane_addr + kColDo + bb2 * 32 + 16, d1);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&do_free[bb2]);
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          d[u] = d0[u];
          d[16 + u] = d1[u];
        }
        const float* rg = ring + bb2 * 8;
#pragma unroll
        for (int r = 0; r < kRowsTc; ++r) {
          // column (r, limb) = 2 r + limb in each value-limb chain
          const float hi = static_cast<float>(static_cast<int>(d[2 * r])) +
                           static_cast<float>(static_cast<int>(d[2 * r + 1])) * (1.f / 128.f);
          const float lo = static_cast<float>(static_cast<int>(d[16 + 2 * r])) +
                           static_cast<float>(static_cast<int>(d[16 + 2 * r + 1])) * (1.f / 128.f);
          acc[r] = acc[r] * rg[r] + v_scale * rg[4 + r] * (hi + lo * (1.f / 128.f));
        }
        return true;
      };
      for (int tj = 0; tj < nt_tiles; ++tj, ++j) {
        const int b = j & 1;
        const int64_t t0 = tb + int64_t(tj) * kTT;
        const int nt = static_cast<int>((te - t0 < kTT) ? te - t0 : kTT);
        const bool valid = lrow < nt;
        float kn = 0.f, rn = 0.f, vn = 0.f;
        if (valid) {
          kn = __ldg(a.knorm + row0 + t0 + lrow);
          rn = __ldg(a.krnorm + row0 + t0 + lrow);
          vn = __ldg(a.vnorm + row0 + t0 + lrow);
        }
        bool ok = __all_sync(0xffffffffu, mbar_wait(&s_full[b], (j >> 1) & 1));
        tc_fence_after();
        uint32_t d0[16], d1[16], d2[16], d3[16];
        tmem_ld16(lane_addr + kColDs + b * kDsCols, d0);
        tmem_ld16(lane_addr + kColDs + b * kDsCols + 16, d1);
        tmem_ld16(lane_addr + kColDs + b * kDsCols + 32, d2);
        tmem_ld16(lane_addr + kColDs + b * kDsCols + 48, d3);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ds_free[b]);
        float score[kRowsTc];
#pragma unroll
        for (int r = 0; r < kRowsTc; ++r) {
          float c1 = 0.f, c2 = 0.f, c3 = 0.f, sb = 0.f;
#pragma unroll
          for (int l = 2; l >= 0; --l) {
            c1 = c1 * (1.f / 128.f) + static_cast<float>(static_cast<int>(d0[3 * r + l]));
            c2 = c2 * (1.f / 128.f) + static_cast<float>(static_cast<int>(d1[3 * r + l]));
            c3 = c3 * (1.f / 128.f) + static_cast<float>(static_cast<int>(d2[3 * r + l]));
            sb = sb * (1.f / 128.f) + static_cast<float>(static_cast<int>(d3[3 * r + l]));
          }
          const float mse = k_scale * isc[r] * (c1 + (c2 + c3 * (1.f / 128.f)) * (1.f / 128.f));
          const float qjl = 2.f * isc[4 + r] * sb - isc[8 + r];
          score[r] = valid ? a.scale * (kn * mse + alpha * rn * qjl) : -INFINITY;
        }
        if (a.scores_out && valid) {
#pragma unroll
          for (int r = 0; r < kRowsTc; ++r) a.scores_out[qrow[r] * sh.n_ctx + t0 + lrow] = score[r];
        }
        // Online softmax over the tile.
#pragma unroll
        for (int r = 0; r < kRowsTc; ++r) {
          const float mx = warp_max(score[r]);
          if (lane == 0) red[cw * 8 + r] = mx;
        }
        if (wg_sync_or(3, !ok || *abort_s != 0)) {
          if (!ok && lane == 0 && cw == 0) fail();
          stop = true;
          break;
        }
        float corr[kRowsTc], p[kRowsTc];
#pragma unroll
        for (int r = 0; r < kRowsTc; ++r) {
          float mx = red[r];
#pragma unroll
          for (int w2 = 1; w2 < 4; ++w2) mx = fmaxf(mx, red[w2 * 8 + r]);
          const float m_new = fmaxf(m_run[r], mx);
          corr[r] = (m_run[r] == -INFINITY) ? 0.f : __expf(m_run[r] - m_new);
          m_run[r] = m_new;
          p[r] = valid ? __expf(score[r] - m_new) : 0.f;
        }
        wg_sync(2);                                // everyone has read the maxima
#pragma unroll
        for (int r = 0; r < kRowsTc; ++r) {
          const float ps = warp_sum(p[r]);
          const float wm = warp_max(p[r] * vn);
          if (lane == 0) {
            red[cw * 8 + r] = ps;
            red[cw * 8 + 4 + r] = wm;
          }
        }
        wg_sync(2);
        float sp[kRowsTc];
#pragma unroll
        for (int r = 0; r < kRowsTc; ++r) {
          float ps = 0.f, wm = 0.f;
#pragma unroll
          for (int w2 = 0; w2 < 4; ++w2) {
            ps += red[w2 * 8 + r];
            wm = fmaxf(wm, red[w2 * 8 + 4 + r]);
          }
          l_run[r] = l_run[r] * corr[r] + ps;
          sp[r] = wm > 0.f ? wm / 127.f : 1.f;
        }
        // Publish this tile's correction and weight scale for its value epilogue.
        if (lrow < kRowsTc) {
#pragma unroll
          for (int r = 0; r < kRowsTc; ++r)
            if (r == lrow) {
              ring[b * 8 + r] = corr[r];
              ring[b * 8 + 4 + r] = sp[r];
            }
        }
        // Weight limbs into the P tile (row 2 r + limb, column = token).
        if (!__all_sync(0xffffffffu, mbar_wait(&p_free[b], ((j >> 1) & 1) ^ 1)) && lane == 0) fail();
        unsigned char* pt = sm + Sm::kOffP + b * 2048;
#pragma unroll
        for (int r = 0; r < kRowsTc; ++r) {
          const float x = p[r] * vn / sp[r];
          const int l0 = __float2int_rn(x);
          const int l1 = __float2int_rn((x - static_cast<float>(l0)) * 128.f);
          pt[sw_byte(2 * r, lrow)] = static_cast<unsigned char>(static_cast<int8_t>(l0));
          pt[sw_byte(2 * r + 1, lrow)] = static_cast<unsigned char>(static_cast<int8_t>(l1));
        }
#pragma unroll
        for (int n = 8; n < 16; ++n) pt[sw_byte(n, lrow)] = 0;
        fence_proxy_async_smem();
        wg_sync(2);                                // ring + red reads done before reuse
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[b]);
        // Fold the previous tile's values (its correction comes first).
        if (tj >= 1 && !value_epilogue(j - 1)) {
          if (lane == 0) fail();
        }
      }
      if (stop) break;
      // Last tile of the item, then the partials.
      if (!value_epilogue(j - 1) && lane == 0) fail();
      const int64_t pbase = (int64_t(split)) * (kD + 2);
#pragma unroll
      for (int r = 0; r < kRowsTc; ++r) {
        float* pr = a.part + qrow[r] * sh.n_splits * (kD + 2) + pbase;
        pr[lrow] = acc[r];
        if (lrow == 0) {
          pr[kD] = m_run[r];
          pr[kD + 1] = l_run[r];
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
    if (lane == 0) {
      umma_commit(drain);
      mbar_wait(drain, 0);
    }
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
