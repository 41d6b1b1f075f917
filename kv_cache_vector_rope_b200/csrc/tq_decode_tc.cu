// Fused tensor-core decode attention (sm_100a, tcgen05 kind::i8) for d = 128,
// four query rows per KV stream (a GQA group of four heads, one query each),
// 3-bit values and 2-4-bit keys: the whole call in two launches (a query-side
// prologue and the main kernel) after a memset of the arrival counters.
//
// Sources: gist.science "TurboESM ..." section 2E (one fused kernel unpacks
// the codes, applies the QJL correction and the inverse rotation and runs an
// online softmax, with no dequantised tensor in memory) and 7minutos.es
// "KV cache ... TurboQuant" Etapa 2 (the QJL estimator).
//
//   Work        all (stream, 128-token tile) pairs in stream order are cut into
//               equal contiguous ranges, one per persistent CTA (longer than
//               512 tiles: cut again). A range splits into segments at stream
//               ends; each segment leaves one partial record (m, l, acc) per
//               query row.
//   Prologue    a small kernel before the main one: per stream q_rot =
//               Pi_K RoPE(q), s = S q_rot and their int8 limbs as the B
//               operands of the score MMAs; the main kernel's loader copies a
//               segment's share in with one bulk copy.
//   Scores      A (TMEM, one lane per token): the key codebook value of every
//               coordinate as three int8 limbs, c = sc (a1 + a2/128 + a3/128^2),
//               and the sign chunk, masked in place (byte 16 j + b = byte b of
//               the sign row AND 1 << j); B (smem): limbs of q_rot and of
//               s' = s 2^-(i mod 8). Limb products of equal weight share an
//               int32 column: 16 MMAs (M = 128, N = 16, K = 32) per tile.
//   Softmax     thread = token. The running maximum m of each query row is set
//               by the segment's first tile and only moves when a weight
//               x = 2^(score - m) ||v|| / V0 (V0: largest ||v|| of that first
//               tile) would exceed 64; then it moves by whole octaves. The
//               weights are 32-bit fixed point, X = rint(x 2^24): their four
//               bytes are the unsigned B limbs of the value MMAs, one 16-byte
//               shared store per token (B MN-major, 16 bytes per token).
//   Values      A (smem, MN-major): the value codebook as two int8 limbs per
//               coordinate, one 128-byte row per token. The PV products add up
//               in TMEM over all tiles of a segment; only when m moves (rare)
//               is the accumulator folded into registers (thread = coordinate)
//               and restarted in the other TMEM region.
//   Combine     the last segment of a stream to finish (a per-stream arrival
//               counter) merges the stream's records and applies Pi_V^T.
// Roles (640 threads, one CTA per SM):
//   warp 0        bulk copies: the index and sign planes into a 4-stage ring,
//                 each segment's query side into one of two copies
//   warp 1        TMEM owner and score MMA issuer   (warp-uniform loop, elected lane)
//   warp 2        PV MMA issuer
//   warp 3        the codebook limb tables (prologue only)
//   warps 4-11    two key groups, alternate tiles: key operands into TMEM and
//                 value operands into smem        (thread = token)
//   warps 12-19   two softmax groups, alternate tiles of a segment: scores,
//                 softmax, weights, folds; together the arrival and the combine
//                 (thread = token / coordinate)
// Every wait is bounded (2 s; the pipeline waits take the launch's limit, which
// the environment variable TQ_TEST_WAIT_NS can shorten); a timeout sets
// TQ_DEV_TIMEOUT and the CTA drains its copies and MMAs (full 2 s limit)
// before it frees TMEM and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "tq_decode_tc.h"
#include "tq_device.cuh"
#include "tq_internal.h"
#include "tq_sm100.cuh"

namespace tq {
namespace {

using namespace sm100;
using dev::load_elem;
using dev::warp_max;
using dev::warp_sum;

constexpr int kD = 128;
constexpr int kTT = 128;               // tokens per tile
constexpr int kStages = 4;
constexpr int kNVh = 3;                // value operand / P buffers (tile j uses j % 3)
// Per stream, the query side of the score MMAs (written by the prologue
// kernel): the B tiles B1 | B2 | B3 | Bs (4 x 2 KB, K-major, 128-byte swizzle)
// and 16 floats: scale*sq[4], 2*ss[4], sum s[4], pad.
constexpr int kQPrepBytes = 4 * 2048 + 64;
constexpr int kQPrepStride = 8448;      // bytes between streams in the workspace (256-aligned)
constexpr int kBStride = 9216;          // bytes between the two smem copies (1024-aligned)
constexpr int kThreads = 640;          // 20 warps
constexpr int kRows = 4;               // query rows per stream
constexpr int kMaxSegTiles = 512;      // PV accumulators: < 2^31 over this many tiles
constexpr int kMaxGrid = 256;
constexpr int kRecFloats = 132;        // partial record: acc[128], m, l, pad
constexpr int kWLoader = 0, kWScore = 1, kWPv = 2, kWKey0 = 4, kWVs0 = 12;   // key groups 4-7, 8-11; value+softmax groups 12-15, 16-19

// TMEM columns (32-bit): A_score x2 at 0, 128 (a1 | a2 | a3 | sgn, 32 each);
// D_score x2 at 256, 288 (mse 16 | sgn 16); D_o regions x4 at 320 + 32 X
// (two per softmax group; two value-limb chains of 16 columns each).
constexpr uint32_t kColA = 0, kColDs = 256, kColDo = 320, kTmemCols = 512;

// Instruction descriptor, kind::i8: s32 D, M = 128, N = 16.
__host__ __device__ constexpr uint32_t idesc_i8(bool a_signed, bool a_mn_major, bool b_mn_major, bool b_signed) {
  return (2u << 4) | ((a_signed ? 1u : 0u) << 7) | ((b_signed ? 1u : 0u) << 10) | ((a_mn_major ? 1u : 0u) << 15) |
         ((b_mn_major ? 1u : 0u) << 16) | ((16u >> 3) << 17) | ((128u >> 4) << 24);
}

template <int KB>
struct FSm {
  static constexpr int kRbk = kD * KB / 8;
  static constexpr int kOffKs = kTT * kRbk;                        // sign rows within a stage
  static constexpr int kOffVi = kOffKs + kTT * 16;                 // value index rows
  static constexpr int kStageBytes = kOffVi + kTT * 48;
  static constexpr int kStageStride = ((kStageBytes + 1023) / 1024) * 1024;
  static constexpr int kOffVh = kStages * kStageStride;            // kNVh buffers x 2 limbs x 16 KB
  static constexpr int kVhBytes = 2 * kTT * 128;
  static constexpr int kOffP = kOffVh + kNVh * kVhBytes;           // kNVh x [128 tokens][16 B]
  static constexpr int kOffB = kOffP + kNVh * 2048;                // 2 segments x (B1 | B2 | B3 | Bs | consts)
  static constexpr int kOffQ = kOffB + 2 * kBStride;               // qx, qr, sv: [4][128] floats each (combine)
  static constexpr int kOffPP = kOffQ + 3 * kRows * kD * 4;        // [4][128] floats: matvec partials
  static constexpr int kOffRed = kOffPP + kRows * kD * 4;          // [16][16] floats
  static constexpr int kOffNrm = kOffRed + 16 * 16 * 4;            // [2 groups][4 slots][3][128] norms
  static constexpr int kOffRec = kOffNrm + 2 * 4 * 3 * kTT * 4;    // [8][16] words: tile records
  static constexpr int kOffTab = kOffRec + 8 * 16 * 4;             // limb tables (20 words) + 2 scales
  static constexpr int kOffBar = kOffTab + 32 * 4;
  static constexpr int kNumBars = 2 * kStages + 5 * 2 + 2 * kNVh + 4 + 4 + 2;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kBytes = kOffMisc + 64 + 1024;               // + alignment slack
};

static_assert(FSm<4>::kBytes <= 232448, "shared memory plan exceeds 227 KB");

struct FusedArgs {
  DecodeArgs v;
  int64_t T, Ts;       // tiles in all, tiles per stream
  int V;               // virtual CTAs
  int* counters;       // [streams] arrivals (zero at launch)
  unsigned char* qprep;  // [streams][kQPrepStride] query side of the score MMAs
  uint64_t wait_ns;    // pipeline wait limit (drains keep 2 s)
};

// int8 limbs of the key codebook (three) and the value codebook (two),
// c ~ scale (a1 + a2/128 + a3/128^2) with scale = max|c| / 127, as byte tables
// (byte k of word k/4 = code k): tab[0..3] a1, [4..7] a2, [8..11] a3 (keys),
// [12..15] a1, [16..19] a2 (values). One warp: lane k < nk takes key code k,
// lane 16 + k value code k; fp64, so every CTA derives the same tables.
__device__ void codebook_limbs_warp(const float* cK, int nk, const float* cV, uint32_t* tab, float* scales, int lane) {
  const bool key = lane < 16, has = key ? lane < nk : lane < 24;
  const int k = key ? lane : lane - 16;
  const double c = has ? static_cast<double>(__ldg((key ? cK : cV) + k)) : 0.0;
  double m = fabs(c);
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) m = fmax(m, __shfl_xor_sync(0xffffffffu, m, o));   // within each half
  const double sc = m > 0.0 ? m / 127.0 : 1.0;
  if (lane < 20) tab[lane] = 0u;
  __syncwarp();
  if (has) {
    unsigned char* tb = reinterpret_cast<unsigned char*>(tab) + (key ? 0 : 48);
    const double r0 = c / sc;
    const double a1 = rint(r0);
    const double r1 = (r0 - a1) * 128.0;
    const double a2 = rint(r1);
    tb[k] = static_cast<unsigned char>(static_cast<int8_t>(a1));
    tb[16 + k] = static_cast<unsigned char>(static_cast<int8_t>(a2));
    if (key) tb[32 + k] = static_cast<unsigned char>(static_cast<int8_t>(rint((r1 - a2) * 128.0)));
  }
  if (lane == 0) scales[0] = static_cast<float>(sc);
  if (lane == 16) scales[1] = static_cast<float>(sc);
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
// One lane of the (converged) warp; the others get false.
__device__ __forceinline__ bool elect_one() {
  uint32_t p;
  asm volatile(
      "{\n\t.reg .pred P;\n\t.reg .b32 r;\n\t"
      "elect.sync r|P, 0xffffffff;\n\t"
      "selp.u32 %0, 1, 0, P;\n\t}"
      : "=r"(p));
  return p != 0;
}

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
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src, uint32_t n) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void named_sync(int id, int n) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory"); }
// Shared-memory descriptor of an MN-major operand without swizzle whose
// rows (one per K index) are 16 bytes: core matrices of 8 rows x 16 B, 128 B
// apart along K.
__device__ __forceinline__ uint64_t desc_mn_noswz(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>(128u >> 4) << 16;     // LBO
  d |= static_cast<uint64_t>(128u >> 4) << 32;     // SBO
  d |= static_cast<uint64_t>(1u) << 46;            // descriptor version for sm_100
  return d;                                        // layout 0: no swizzle
}

// y[r][i] = sum_j M[i][j] x[r][j] for four rows (x, y: shared [4][128]) on
// 256 threads: thread u takes output coordinate i = u % 128 and the input
// coordinates of half u / 128 (64 of them, 16 float4s), with all of its row
// loads in flight; the two partial sums meet in pp [2][4][128]. Two barriers
// of the 256 threads (id 2).
__device__ __forceinline__ void matvec4_split(const float* __restrict__ M, const float* x, float* y, float* pp, int u) {
  const int i = u & 127, part = u >> 7;
  const float4* row = reinterpret_cast<const float4*>(M + int64_t(i) * kD) + part * 16;
  float4 mv[16];
#pragma unroll
  for (int k = 0; k < 16; ++k) mv[k] = __ldg(row + k);
  float acc[kRows] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int k = 0; k < 16; ++k) {
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
      const float4 xv = reinterpret_cast<const float4*>(x + r * kD)[part * 16 + k];
      acc[r] = fmaf(mv[k].x, xv.x, fmaf(mv[k].y, xv.y, fmaf(mv[k].z, xv.z, fmaf(mv[k].w, xv.w, acc[r]))));
    }
  }
  if (part == 1) {
#pragma unroll
    for (int r = 0; r < kRows; ++r) pp[r * kD + i] = acc[r];
  }
  named_sync(2, 256);
  if (part == 0) {
#pragma unroll
    for (int r = 0; r < kRows; ++r) y[r * kD + i] = acc[r] + pp[r * kD + i];
  }
  named_sync(2, 256);
}

// Work partition: all (stream, tile) pairs in stream order, cut into V equal
// contiguous ranges ("virtual CTAs", V >= grid); physical CTA c takes v = c,
// c + grid, ... A range splits at stream ends into segments; the segment of
// virtual CTA v in stream s owns partial record v + s (the pair is unique
// because both the ranges and the streams are ordered).
struct Part {
  int64_t T;      // tiles in all
  int64_t Ts;     // tiles per stream
  int V;          // virtual CTAs
};
__device__ __forceinline__ int64_t vstart(const Part& p, int64_t v) { return (v * p.T) / p.V; }
// Virtual CTA holding global tile g.
__device__ __forceinline__ int64_t vof(const Part& p, int64_t g) {
  int64_t v = (g * p.V) / p.T;
  while (v > 0 && vstart(p, v) > g) --v;
  while (v + 1 < p.V && vstart(p, v + 1) <= g) ++v;
  return v;
}

struct Seg {
  int64_t v, s;        // virtual CTA, stream
  int64_t t0, t1;      // tiles [t0, t1) of the stream
  int idx;             // segment number within this CTA
};
// Segments of this CTA, in order (every role walks the same sequence).
struct SegIter {
  Part p;
  int64_t v, g, g1;
  int idx;
  __device__ SegIter(const Part& pp) : p(pp), v(blockIdx.x), g(0), g1(0), idx(0) {
    if (v < p.V) {
      g = vstart(p, v);
      g1 = vstart(p, v + 1);
    }
  }
  __device__ bool next(Seg& sg) {
    while (v < p.V && g >= g1) {
      v += gridDim.x;
      if (v < p.V) {
        g = vstart(p, v);
        g1 = vstart(p, v + 1);
      }
    }
    if (v >= p.V) return false;
    const int64_t s = g / p.Ts;
    const int64_t ge = min(g1, (s + 1) * p.Ts);
    sg.v = v;
    sg.s = s;
    sg.t0 = g - s * p.Ts;
    sg.t1 = ge - s * p.Ts;
    sg.idx = idx++;
    g = ge;
    return true;
  }
};

// ---------------------------------------------------------------------------
// Query side of the score MMAs, one CTA of 256 threads per KV stream (runs
// before the main kernel): q' = RoPE(q), q_rot = Pi_K q', s = S q_rot for the
// stream's four query rows, then their int8 limbs as the B tiles
//   B1/B2/B3  rows 4 r + w hold limb w, w-1, w-2 of q_rot row r / sq_r
//   Bs        rows 4 r + l hold limb l of s'_i = s_i 2^-(i mod 8) / ss_r at K
//             position 16 (i mod 8) + i / 8
// (K-major, 128-byte swizzle, 2 KB each) and the row constants scale * sq_r,
// 2 ss_r and sum_i s_i (sq_r = max|q_rot| / 127, ss_r = max|s'| / 127).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) decode_qprep_kernel(FusedArgs A) {
  __shared__ __align__(16) float qx[kRows * kD], qr[kRows * kD], sv[kRows * kD], pp[kRows * kD];
  __shared__ __align__(16) float red[8 * 16];
  __shared__ __align__(1024) unsigned char bt[4 * 2048];
  const DecodeArgs& a = A.v;
  const DecodeShape& sh = a.sh;
  const int u = threadIdx.x, lane = u & 31;
  const int64_t bkv = blockIdx.x;
  const int kv = static_cast<int>(bkv % sh.hkv), bb = static_cast<int>(bkv / sh.hkv);
  const int G = sh.hq / sh.hkv;
  auto qrow = [&](int r) -> int64_t { return int64_t(bb) * sh.hq + kv * G + r; };   // nq == 1
  const bool rope = a.q_pos != nullptr && a.rope_base > 0.0;
  {
    const int r = u >> 6, i = u & 63;
    const int64_t qi = qrow(r) * kD;
    float x0 = load_elem(a.q, a.q_dtype, qi + i), x1 = load_elem(a.q, a.q_dtype, qi + i + kD / 2);
    if (rope) {
      const int pos = a.q_pos[bb];
      if (pos < 0 && a.d_status) atomicOr(a.d_status, TQ_DEV_BAD_POSITION);
      double sn, cs;
      sincos(dev::rope_angle(pos, i, kD, a.rope_base), &sn, &cs);
      const double r0 = double(x0) * cs - double(x1) * sn, r1 = double(x0) * sn + double(x1) * cs;
      x0 = static_cast<float>(r0);
      x1 = static_cast<float>(r1);
    }
    qx[r * kD + i] = x0;
    qx[r * kD + i + kD / 2] = x1;
  }
  named_sync(2, 256);
  matvec4_split(a.PiK + int64_t(kv) * a.pi_stride, qx, qr, pp, u);
  matvec4_split(a.S, qr, sv, pp, u);
  const int i = u & 127, rr = 2 * (u >> 7);
  // Row scales: warp w8 covers row w8 / 2, coordinates of half w8 % 2.
  {
    const int w8 = u >> 5, r = w8 >> 1, i0 = (w8 & 1) * 64 + lane;
    float mq = 0.f, ms = 0.f, ssm = 0.f;
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int ii = i0 + 32 * k;
      const float jsc = __uint_as_float(static_cast<uint32_t>(127 - (ii & 7)) << 23);   // 2^-(i mod 8)
      mq = fmaxf(mq, fabsf(qr[r * kD + ii]));
      ms = fmaxf(ms, fabsf(sv[r * kD + ii]) * jsc);
      ssm += sv[r * kD + ii];
    }
    mq = warp_max(mq);
    ms = warp_max(ms);
    ssm = warp_sum(ssm);
    if (lane == 0) {
      red[w8 * 16 + 0] = mq;
      red[w8 * 16 + 1] = ms;
      red[w8 * 16 + 2] = ssm;
    }
  }
  named_sync(2, 256);
  unsigned char* out = A.qprep + bkv * kQPrepStride;
  {
    float sq[2], ss[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int r = rr + k;
      const float mq = fmaxf(red[(2 * r) * 16 + 0], red[(2 * r + 1) * 16 + 0]);
      const float ms = fmaxf(red[(2 * r) * 16 + 1], red[(2 * r + 1) * 16 + 1]);
      sq[k] = mq > 0.f ? mq / 127.f : 1.f;
      ss[k] = ms > 0.f ? ms / 127.f : 1.f;
    }
    if (u < kRows) {
      const int r = u;
      const float mq = fmaxf(red[(2 * r) * 16 + 0], red[(2 * r + 1) * 16 + 0]);
      const float ms = fmaxf(red[(2 * r) * 16 + 1], red[(2 * r + 1) * 16 + 1]);
      float* qc = reinterpret_cast<float*>(out + 4 * 2048);
      qc[r] = a.scale * (mq > 0.f ? mq / 127.f : 1.f);
      qc[4 + r] = 2.f * (ms > 0.f ? ms / 127.f : 1.f);
      qc[8 + r] = red[(2 * r) * 16 + 2] + red[(2 * r + 1) * 16 + 2];
      qc[12 + r] = 0.f;
    }
    const int ks = 16 * (i & 7) + (i >> 3);
    const float jsc = __uint_as_float(static_cast<uint32_t>(127 - (i & 7)) << 23);
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int r = rr + k;
      int lq[4], ls[4];
      limbs4(qr[r * kD + i] / sq[k], lq);
      limbs4(sv[r * kD + i] * jsc / ss[k], ls);
#pragma unroll
      for (int w2 = 0; w2 < 4; ++w2) {
        bt[sw_byte(4 * r + w2, i)] = static_cast<unsigned char>(static_cast<int8_t>(lq[w2]));
        bt[2048 + sw_byte(4 * r + w2, i)] = static_cast<unsigned char>(static_cast<int8_t>(w2 >= 1 ? lq[w2 - 1] : 0));
        bt[4096 + sw_byte(4 * r + w2, i)] = static_cast<unsigned char>(static_cast<int8_t>(w2 >= 2 ? lq[w2 - 2] : 0));
        bt[6144 + sw_byte(4 * r + w2, ks)] = static_cast<unsigned char>(static_cast<int8_t>(ls[w2]));
      }
    }
  }
  named_sync(2, 256);
  // The tiles leave in 16-byte pieces (swizzled layout kept byte for byte).
#pragma unroll
  for (int k = 0; k < 2; ++k) reinterpret_cast<uint4*>(out)[u + 256 * k] = reinterpret_cast<const uint4*>(bt)[u + 256 * k];
}

template <int KB>
__global__ void __launch_bounds__(kThreads, 1) decode_fused_kernel(FusedArgs A) {
  using Sm = FSm<KB>;
  constexpr int kRbk = Sm::kRbk;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const DecodeArgs& a = A.v;
  const DecodeShape& sh = a.sh;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + Sm::kOffBar);
  uint64_t* st_full = bars;                       // [kStages] loader (tx)
  uint64_t* st_empty = bars + kStages;            // [kStages] the tile's key group read the stage
  uint64_t* a_full = bars + 2 * kStages;          // [2] key group of the buffer
  uint64_t* s_full = a_full + 2;                  // [2] score commit (also frees the A operand)
  uint64_t* ds_free = s_full + 2;                 // [2] the group read the score columns
  uint64_t* pv_ready = ds_free + 2;               // [kNVh] value operand (key group) and P (softmax group) written
  uint64_t* pv_full = pv_ready + kNVh;            // [kNVh] PV commit (frees the value operand and P)
  uint64_t* bt_full = pv_full + kNVh;             // [2] per segment parity: the query-side copy (tx)
  uint64_t* bt_free = bt_full + 2;                // [2] score issuer: the segment's score MMAs are done
  uint64_t* reg_done = bt_free + 2;               // [4] PV commit when a TMEM value region closes
  uint64_t* reg_free = reg_done + 4;              // [4] the owning group folded the region
  uint64_t* drain = reg_free + 4;                 // [2] score issuer, PV issuer
  uint64_t* a_free = s_full;
  uint64_t* vh_free = pv_full;

  uint32_t* tmem_base_s = reinterpret_cast<uint32_t*>(sm + Sm::kOffMisc);
  volatile int* abort_s = reinterpret_cast<volatile int*>(sm + Sm::kOffMisc + 4);
  int* merge_s = reinterpret_cast<int*>(sm + Sm::kOffMisc + 8);
  float* qx = reinterpret_cast<float*>(sm + Sm::kOffQ);             // [4][128] RoPE'd q; merged rows
  float* qr = qx + kRows * kD;                                      // [4][128] q_rot
  float* red = reinterpret_cast<float*>(sm + Sm::kOffRed);          // [16][16]
  float* pp = reinterpret_cast<float*>(sm + Sm::kOffPP);            // [4][128] partial sums
  uint32_t* recs = reinterpret_cast<uint32_t*>(sm + Sm::kOffRec);   // [8][16] tile records
  uint32_t* tab = reinterpret_cast<uint32_t*>(sm + Sm::kOffTab);    // ka1 ka2 ka3 va1 va2 (4 words each)
  float* cb_scale = reinterpret_cast<float*>(sm + Sm::kOffTab + 20 * 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const Part part{A.T, A.Ts, A.V};

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&st_full[s], 1);
      mbar_init(&st_empty[s], 4);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&a_full[b], 4);
      mbar_init(&s_full[b], 1);
      mbar_init(&ds_free[b], 4);

      mbar_init(&bt_full[b], 1);
      mbar_init(&bt_free[b], 1);
      mbar_init(&drain[b], 1);
    }
    for (int x = 0; x < kNVh; ++x) {
      mbar_init(&pv_ready[x], 8);
      mbar_init(&pv_full[x], 1);
    }
    for (int x = 0; x < 4; ++x) {
      mbar_init(&reg_done[x], 1);
      mbar_init(&reg_free[x], 4);
    }
    *abort_s = 0;
    for (int k = 0; k < 8; ++k) recs[k * 16] = 0xFFFFFFFFu;
    mbar_fence_init();
  }
  if (warp == 3) codebook_limbs_warp(a.cK, 1 << sh.kbits, a.cV, tab, cb_scale, lane);
  if (warp == kWScore) {
    tmem_alloc(tmem_base_s, kTmemCols);
    tmem_relinquish();
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
  const int G = sh.hq / sh.hkv;

  if (warp == kWLoader) {
    // ------------------------------------------------------------- loader
    if (lane == 0) {
      int j = 0;
      int bt_last[2] = {0, 0};                   // 1 + index of the last segment copied into each copy
      bool ok = true;
      SegIter it(part);
      Seg sg;
      while (ok && it.next(sg)) {
        const int64_t row0 = sg.s * sh.ctx_stride;
        {
          // The segment's query side (B tiles and row constants) into copy ib,
          // once the score MMAs of segment idx - 2 are done with it.
          const int ib = sg.idx & 1;
          if (*abort_s || !mbar_wait(&bt_free[ib], ((sg.idx >> 1) & 1) ^ 1, A.wait_ns)) { ok = false; break; }
          mbar_expect_tx(&bt_full[ib], kQPrepBytes);
          bulk_g2s(sm + Sm::kOffB + ib * kBStride, A.qprep + sg.s * kQPrepStride, kQPrepBytes, &bt_full[ib]);
          bt_last[ib] = sg.idx + 1;
        }
        for (int64_t tt = sg.t0; tt < sg.t1; ++tt, ++j) {
          const int s = j % kStages;
          if (*abort_s || !mbar_wait(&st_empty[s], ((j / kStages) & 1) ^ 1, A.wait_ns)) { ok = false; break; }
          const int64_t t0 = tt * kTT;
          const int nt = static_cast<int>((sh.n_ctx - t0 < kTT ? sh.n_ctx - t0 : int64_t(kTT)));
          const uint32_t bk = nt * kRbk, bs = nt * 16, bv = nt * 48;
          mbar_expect_tx(&st_full[s], bk + bs + bv);
          unsigned char* st = sm + s * Sm::kStageStride;
          bulk_g2s(st, a.kidx + (row0 + t0) * kRbk, bk, &st_full[s]);
          bulk_g2s(st + Sm::kOffKs, a.ksign + (row0 + t0) * 4, bs, &st_full[s]);
          bulk_g2s(st + Sm::kOffVi, a.vidx + (row0 + t0) * 48, bv, &st_full[s]);
        }
      }
      if (!ok && !*abort_s) fail();
      // Drain: the last copy into every stage and into both query-side
      // copies has landed before the CTA exits.
      for (int k = 1; k <= kStages && j - k >= 0; ++k) {
        const int jj = j - k;
        mbar_wait(&st_full[jj % kStages], (jj / kStages) & 1);
      }
      for (int ib = 0; ib < 2; ++ib)
        if (bt_last[ib] > 0) mbar_wait(&bt_full[ib], ((bt_last[ib] - 1) >> 1) & 1);
    }
  } else if (warp == kWScore || warp == kWPv) {
    // ------------------------------------------ MMA issuers (one warp each)
    // The whole warp runs the loop (descriptor arithmetic stays warp-uniform)
    // and one elected lane issues each MMA: issuing from a divergent
    // single-lane branch costs several times more per MMA.
    const bool leader = elect_one();
    const uint32_t id_mse = idesc_i8(true, false, false, true), id_sgn = idesc_i8(false, false, false, true);
    const uint32_t id_v = idesc_i8(true, true, true, false);
    const uint64_t b_desc0 = desc_k_sw128(smem_u32(sm + Sm::kOffB));   // copy ib at + ib * kBStride
    const uint64_t vh_desc0 = desc_k_sw128(smem_u32(sm + Sm::kOffVh));
    const uint64_t p_desc0 = desc_mn_noswz(smem_u32(sm + Sm::kOffP));
    int j = 0;
    bool ok = true;
    // PV: TMEM region in use per softmax group (2 g + bit g of pcur) and the
    // closes per region (byte X of pcl), kept in registers.
    uint32_t pcur = 0u, pcl = 0u;
    SegIter it(part);
    Seg sg;
    while (ok && it.next(sg)) {
      const int ib = sg.idx & 1;
      const int nt_tiles = static_cast<int>(sg.t1 - sg.t0);
      if (warp == kWScore &&
          !__all_sync(0xffffffffu, mbar_wait(&bt_full[ib], (sg.idx >> 1) & 1, A.wait_ns))) { ok = false; break; }
      for (int tj = 0; tj < nt_tiles; ++tj, ++j) {
        const int b = j & 1;
        const uint32_t ph = (j >> 1) & 1;
        if (__any_sync(0xffffffffu, *abort_s != 0)) { ok = false; break; }
        if (warp == kWScore) {
          const bool w = mbar_wait(&a_full[b], ph, A.wait_ns) && mbar_wait(&ds_free[b], ph ^ 1, A.wait_ns);
          if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
          tc_fence_after();
          const uint32_t d = tmem + kColDs + b * 32;
          const uint32_t a0 = tmem + kColA + b * 128;
          // a1, a2, a3 against B1, B2, B3 (limb-shifted q) into the MSE
          // columns, the sign chunk into its own columns.
          const uint64_t bs = b_desc0 + ((ib * kBStride + 3 * 2048) >> 4);
#pragma unroll
          for (int step = 0; step < 12; ++step) {
            const int ch = step >> 2, k = step & 3;
            const uint64_t bq = b_desc0 + ((ib * kBStride + ch * 2048) >> 4);
            if (leader) umma_i8_ts(d, a0 + ch * 32 + k * 8, bq + ((k * 32) >> 4), id_mse, step != 0);
            if (step < 4 && leader) umma_i8_ts(d + 16, a0 + 96 + k * 8, bs + ((k * 32) >> 4), id_sgn, k != 0);
          }
          if (leader) {
            umma_commit(&s_full[b]);
            if (tj == nt_tiles - 1) umma_commit(&bt_free[ib]);   // the query-side copy is free
          }
        } else {
          const int xb = j % kNVh;                  // value operand / P buffer of the tile
          const bool w = mbar_wait(&pv_ready[xb], (j / kNVh) & 1, A.wait_ns);
          if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
          tc_fence_after();
          const bool flip = recs[(j & 7) * 16 + 1] != 0u;
          const int g = tj & 1;                     // softmax group of the tile
          bool fresh = tj == g;                     // the group's first tile of the segment
          if (flip && !fresh) {
            // The group's running maximum moved: close its region (its MMAs
            // so far are tracked by this commit) and continue in its other one.
            const int Xc = 2 * g + static_cast<int>((pcur >> g) & 1u);
            if (leader) umma_commit(&reg_done[Xc]);
            pcl += 1u << (8 * Xc);
            pcur ^= 1u << g;
            fresh = true;
          }
          const int X = 2 * g + static_cast<int>((pcur >> g) & 1u);
          const uint32_t nclose = (pcl >> (8 * X)) & 0xFFu;
          if (fresh && nclose > 0 &&
              !__all_sync(0xffffffffu, mbar_wait(&reg_free[X], (nclose - 1) & 1, A.wait_ns))) { ok = false; break; }
          tc_fence_after();
          const uint32_t d = tmem + kColDo + X * 32;
          const uint64_t pb = p_desc0 + ((xb * 2048) >> 4);
#pragma unroll
          for (int k = 0; k < 4; ++k) {             // 32 tokens per step = 4 atoms of 8 tokens
#pragma unroll
            for (int limb = 0; limb < 2; ++limb) {  // the two limb chains alternate
              const uint64_t ad = vh_desc0 + ((xb * Sm::kVhBytes + limb * kTT * 128 + k * 4096) >> 4);
              if (leader) umma_i8_ss(d + limb * 16, ad, pb + ((k * 512) >> 4), id_v, !(fresh && k == 0));
            }
          }
          if (leader) umma_commit(&pv_full[xb]);
          if (tj >= nt_tiles - 2) {
            // The group's last tile of the segment: close its region; its next
            // segment starts in the other one.
            if (leader) umma_commit(&reg_done[X]);
            pcl += 1u << (8 * X);
            pcur ^= 1u << g;
          }
        }
        __syncwarp();
      }
    }
    if (!ok && leader && !*abort_s) fail();
    // Every MMA this warp issued completes before TMEM is released.
    if (leader) umma_commit(&drain[warp == kWScore ? 0 : 1]);
    __syncwarp();
    mbar_wait(&drain[warp == kWScore ? 0 : 1], 0);
  } else if (warp >= kWKey0 && warp < kWVs0) {
    // ---------------------------------- key operands (TMEM), two groups of 4 warps
    // Key group kg builds the A operand of the tiles with j % 2 == kg (its
    // own TMEM buffer), then their value operand (smem buffer j % 3); it is
    // the only reader of the stage.
    const int kg = (warp - kWKey0) >> 2;
    const int q = warp & 3;                       // lane quadrant
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(q * 32) << 16);
    const int row = q * 32 + lane;                // token = TMEM lane this thread writes
    uint32_t k1[4], k2[4], k3[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      k1[u] = tab[u];
      k2[u] = tab[4 + u];
      k3[u] = tab[8 + u];
    }
    const uint32_t v1t[2] = {tab[12], tab[13]}, v2t[2] = {tab[16], tab[17]};
    int j = 0;
    bool stop = false;
    SegIter it(part);
    Seg sg;
    while (!stop && it.next(sg)) {
      const int nt_tiles = static_cast<int>(sg.t1 - sg.t0);
      for (int tj = 0; tj < nt_tiles; ++tj, ++j) {
        const int s = j % kStages;
        const int b = j & 1;
        if (b != kg) continue;
        if (!__all_sync(0xffffffffu, mbar_wait(&st_full[s], (j / kStages) & 1, A.wait_ns))) {
          if (lane == 0) fail();
          stop = true;
          break;
        }
        // The row's code words stay in shared memory until the limbs are
        // built (read KB words per 32 coordinates, value codes 3 words per 32);
        // the stage is released after the last read. (Loops are not unrolled:
        // the kernel's five roles share the instruction cache.)
        const unsigned char* st = sm + s * Sm::kStageStride;
        const uint32_t* wrow = reinterpret_cast<const uint32_t*>(st + row * kRbk);
        const uint4 sg4 = reinterpret_cast<const uint4*>(st + Sm::kOffKs + row * 16)[0];
        if (!__all_sync(0xffffffffu, mbar_wait(&a_free[b], ((j >> 1) & 1) ^ 1, A.wait_ns))) {
          if (lane == 0) fail();
          stop = true;
          break;
        }
        tc_fence_after();
        const uint32_t acol = lane_addr + kColA + b * 128;
        // 32 coordinates per step (KB words of codes): nibble selectors, then
        // the three limbs of each coordinate by byte permutes into 8 TMEM
        // columns per limb.
#pragma unroll 1
        for (int qq = 0; qq < 4; ++qq) {
          uint32_t xq[KB + 1];
#pragma unroll
          for (int u = 0; u < KB; ++u) xq[u] = wrow[qq * KB + u];
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
        }
        {
          uint32_t v[32];
          // Sign chunk: column 4 m + u = sign word u AND (0x01010101 << m).
          const uint32_t swd[4] = {sg4.x, sg4.y, sg4.z, sg4.w};
#pragma unroll
          for (int m = 0; m < 8; ++m)
#pragma unroll
            for (int u = 0; u < 4; ++u) v[4 * m + u] = swd[u] & (0x01010101u << m);
          tmem_st32(acol + 96, v);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&a_full[b]);
        // -- value operand of the tile (thread = token): two int8 limbs of the
        // value codebook, one 128-byte M-major row per token and limb, into
        // buffer xb = j % 3 once the product of tile j - 3 has read it.
        const int xb = j % kNVh;
        if (!__all_sync(0xffffffffu, mbar_wait(&vh_free[xb], ((j / kNVh) & 1) ^ 1, A.wait_ns))) {
          if (lane == 0) fail();
          stop = true;
          break;
        }
        {
          const uint32_t* vrow = reinterpret_cast<const uint32_t*>(st + Sm::kOffVi + row * 48);
          unsigned char* vh = sm + Sm::kOffVh + xb * Sm::kVhBytes;
          const int atom = row >> 3, r8 = row & 7;
#pragma unroll 1
          for (int c2 = 0; c2 < 4; ++c2) {
            const uint32_t x4[4] = {vrow[3 * c2], vrow[3 * c2 + 1], vrow[3 * c2 + 2], 0u};
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
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&st_empty[s]);
          mbar_arrive(&pv_ready[xb]);
        }
      }
    }
  } else if (warp >= kWVs0) {
    // ---------------------------------------------- softmax groups (2 x 4 warps)
    // Group g takes the segment's tiles tj with tj % 2 == g: it turns their
    // scores into weights and folds its own TMEM regions (2g, 2g + 1). Both
    // groups share the arrival and the combine (256 threads on barrier 2).
    const int grp = (warp - kWVs0) >> 2;          // 0 or 1
    const int gbar = grp == 0 ? 1 : 4;            // the group's named barrier (128 threads)
    const int u = tid - kWVs0 * 32;               // 0..255
    const int q = warp & 3;                       // lane quadrant
    const int lrow = q * 32 + lane;               // token (TMEM lane) / coordinate
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(q * 32) << 16);
    const float alpha = static_cast<float>(dev::kSqrtHalfPi / kD);
    constexpr float kLog2e = 1.4426950408889634f;
    int j = 0;                                    // CTA-local tile counter
    bool stop = false;
    uint32_t gcur = 0u;                           // region in use: 2 grp + gcur
    uint32_t gcl = 0u;                            // closes of the group's two regions (byte each)
    float* nring = reinterpret_cast<float*>(sm + Sm::kOffNrm) + grp * (4 * 3 * kTT);
    SegIter it(part);
    Seg sg;
    while (it.next(sg)) {
      const int ib = sg.idx & 1;
      const int nt_tiles = static_cast<int>(sg.t1 - sg.t0);
      const int64_t bkv = sg.s;                   // stream = b * hkv + kv
      const int kv = static_cast<int>(bkv % sh.hkv), bb = static_cast<int>(bkv / sh.hkv);
      const int64_t row0 = bkv * sh.ctx_stride;
      const int64_t te = (sg.t1 * kTT < sh.n_ctx ? sg.t1 * kTT : sh.n_ctx);
      const int j0 = j;
      auto qrow = [&](int r) -> int64_t { return int64_t(bb) * sh.hq + kv * G + r; };   // nq == 1
      // Norms of the group's k-th tile (tile 2k + grp) go into ring slot k % 4,
      // three tiles ahead, by cp.async (one commit group per tile).
      auto norm_fetch = [&](int k) {
        const int tj = 2 * k + grp;
        if (tj < nt_tiles) {
          const int64_t t = (sg.t0 + tj) * kTT + lrow;
          const bool ok = t < te;
          const int64_t off = row0 + (ok ? t : 0);
          const uint32_t n = ok ? 4u : 0u;
          float* slot = nring + (k & 3) * (3 * kTT);
          cp_async4(smem_u32(slot + lrow), a.knorm + off, n);
          cp_async4(smem_u32(slot + kTT + lrow), a.krnorm + off, n);
          cp_async4(smem_u32(slot + 2 * kTT + lrow), a.vnorm + off, n);
        }
        cp_async_commit();
      };
      norm_fetch(0);
      norm_fetch(1);
      norm_fetch(2);
      // ---------------- the segment's query side (copied in by the loader)
      if (!__all_sync(0xffffffffu, mbar_wait(&bt_full[ib], (sg.idx >> 1) & 1, A.wait_ns)) && lane == 0) fail();
      const float* qc = reinterpret_cast<const float*>(sm + Sm::kOffB + ib * kBStride + 4 * 2048);
      // ---------------- the group's tiles
      float kq[kRows], ks2[kRows], ssum[kRows];
#pragma unroll
      for (int r = 0; r < kRows; ++r) {
        kq[r] = qc[r] * k_scale;
        ks2[r] = qc[4 + r];
        ssum[r] = qc[8 + r];
      }
      const float kr = a.scale * alpha;
      float m_run[kRows], l_part[kRows], acc[kRows], m_acc[kRows];
#pragma unroll
      for (int r = 0; r < kRows; ++r) {
        m_run[r] = -INFINITY;
        l_part[r] = 0.f;
        acc[r] = 0.f;
        m_acc[r] = -INFINITY;
      }
      float v0 = 0.f, inv_v0 = 0.f;
      // Folds the group's current region (closed by the PV issuer; running
      // maxima m_seg in effect for its tiles) into acc (thread = coordinate),
      // then moves to the other region.
      auto fold = [&](const float (&m_seg)[kRows]) -> bool {
        const int X = 2 * grp + static_cast<int>(gcur);
        const uint32_t nclose = (gcl >> (8 * gcur)) & 0xFFu;
        if (!__all_sync(0xffffffffu, mbar_wait(&reg_done[X], nclose & 1, A.wait_ns))) return false;
        tc_fence_after();
        uint32_t dv[32];
        tmem_ld32(lane_addr + kColDo + X * 32, dv);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&reg_free[X]);
        gcl += 1u << (8 * gcur);
        gcur ^= 1u;
#pragma unroll
        for (int r = 0; r < kRows; ++r) {
          float w0 = 0.f, w1 = 0.f;
#pragma unroll
          for (int w8 = 3; w8 >= 0; --w8) {
            w0 = fmaf(w0, 256.f, static_cast<float>(static_cast<int32_t>(dv[4 * r + w8])));
            w1 = fmaf(w1, 256.f, static_cast<float>(static_cast<int32_t>(dv[16 + 4 * r + w8])));
          }
          const float val = v_scale * fmaf(w1, 1.f / 128.f, w0) * (1.f / 16777216.f);
          const float c = (m_acc[r] == -INFINITY) ? 0.f : ex2(m_acc[r] - m_seg[r]);
          acc[r] = fmaf(acc[r], c, val);
          m_acc[r] = m_seg[r];
        }
        return true;
      };
      for (int k = 0; 2 * k + grp < nt_tiles; ++k) {
        const int tj = 2 * k + grp;
        const int jt = j0 + tj;
        const int b = jt & 1;
        const int64_t t0 = (sg.t0 + tj) * kTT;
        const int nt = static_cast<int>((sh.n_ctx - t0 < kTT ? sh.n_ctx - t0 : int64_t(kTT)));
        const bool valid = lrow < nt;
        norm_fetch(k + 3);
        // -- scores of the tile (thread = token)
        cp_async_wait<3>();
        const float* slot = nring + (k & 3) * (3 * kTT);
        const float kn = slot[lrow], rn = slot[kTT + lrow], vn = slot[2 * kTT + lrow];
        const bool ok = __all_sync(0xffffffffu, mbar_wait(&s_full[b], (jt >> 1) & 1, A.wait_ns));
        tc_fence_after();
        // MSE part: weights 1, 1/128, 1/128^2 of the key-limb products
        // (weight 3 is below 1e-6 of the first); sign part: four limbs.
        // The two halves are read one after the other (fewer live registers).
        float mse[kRows], sgn[kRows];
        {
          uint32_t d[16];
          tmem_ld16(lane_addr + kColDs + b * 32, d);
          tmem_ld_wait();
#pragma unroll
          for (int r = 0; r < kRows; ++r) {
            const int32_t m01 = static_cast<int32_t>(d[4 * r]) * 128 + static_cast<int32_t>(d[4 * r + 1]);
            mse[r] = fmaf(static_cast<float>(static_cast<int32_t>(d[4 * r + 2])), 1.f / 16384.f,
                          static_cast<float>(m01) * (1.f / 128.f));
          }
          tmem_ld16(lane_addr + kColDs + b * 32 + 16, d);
          tmem_ld_wait();
#pragma unroll
          for (int r = 0; r < kRows; ++r) {
            const int32_t e01 = static_cast<int32_t>(d[4 * r]) * 128 + static_cast<int32_t>(d[4 * r + 1]);
            const int32_t e23 = static_cast<int32_t>(d[4 * r + 2]) * 128 + static_cast<int32_t>(d[4 * r + 3]);
            sgn[r] = fmaf(static_cast<float>(e23), 1.f / 2097152.f, static_cast<float>(e01) * (1.f / 128.f));
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ds_free[b]);
        float s2[kRows];
#pragma unroll
        for (int r = 0; r < kRows; ++r) {
          const float qjl = fmaf(ks2[r], sgn[r], -ssum[r]);
          const float sn = fmaf(kq[r] * kn, mse[r], kr * rn * qjl);
          if (a.scores_out && valid) a.scores_out[qrow(r) * sh.n_ctx + t0 + lrow] = sn;
          s2[r] = valid ? sn * kLog2e : -INFINITY;
        }
        bool flip = false;
        float m_old[kRows];
#pragma unroll
        for (int r = 0; r < kRows; ++r) m_old[r] = m_run[r];
        float x[kRows], p[kRows];
        if (k == 0) {
          // The group's first tile sets its running maxima and V0.
#pragma unroll
          for (int r = 0; r < kRows; ++r) {
            const float mx = warp_max(s2[r]);
            if (lane == 0) red[(8 + 4 * grp + q) * 16 + r] = mx;
          }
          {
            const float vm = warp_max(valid ? vn : 0.f);
            if (lane == 0) red[(8 + 4 * grp + q) * 16 + 4] = vm;
          }
          named_sync(gbar, 128);
          v0 = 0.f;
#pragma unroll
          for (int w2 = 0; w2 < 4; ++w2) v0 = fmaxf(v0, red[(8 + 4 * grp + w2) * 16 + 4]);
#pragma unroll
          for (int r = 0; r < kRows; ++r) {
            float mx = red[(8 + 4 * grp) * 16 + r];
#pragma unroll
            for (int w2 = 1; w2 < 4; ++w2) mx = fmaxf(mx, red[(8 + 4 * grp + w2) * 16 + r]);
            m_run[r] = mx;
            m_old[r] = mx;
          }
          inv_v0 = v0 > 0.f ? 1.f / v0 : 0.f;
          named_sync(gbar, 128);
        }
        const float wv = vn * inv_v0;
        bool need = false;
#pragma unroll
        for (int r = 0; r < kRows; ++r) {
          p[r] = valid ? ex2(fminf(s2[r] - m_run[r], 100.f)) : 0.f;
          x[r] = p[r] * wv;
          need |= !(x[r] <= 64.f) && valid;
        }
        // One vote per tile (uniform over the group's four warps): a weight
        // out of range, or a failed wait / abort anywhere in the group.
        const bool bad = !ok || *abort_s != 0;
        if (wg_sync_or(gbar, need || bad)) {
          if (wg_sync_or(gbar, bad)) {
            if (!ok && lane == 0) fail();
            stop = true;
            break;
          }
          // A weight would leave the fixed-point range: move the running
          // maximum by the whole number of octaves that brings every weight
          // of the tile back to <= 1.
#pragma unroll
          for (int r = 0; r < kRows; ++r) {
            const float z = valid ? (s2[r] - m_run[r]) + __log2f(fmaxf(wv, 1e-30f)) : -INFINITY;
            const float zm = warp_max(z);
            if (lane == 0) red[(8 + 4 * grp + q) * 16 + r] = zm;
          }
          named_sync(gbar, 128);
#pragma unroll
          for (int r = 0; r < kRows; ++r) {
            float zm = red[(8 + 4 * grp) * 16 + r];
#pragma unroll
            for (int w2 = 1; w2 < 4; ++w2) zm = fmaxf(zm, red[(8 + 4 * grp + w2) * 16 + r]);
            const float dl = zm > 0.f ? ceilf(zm) : 0.f;
            m_run[r] += dl;
            l_part[r] *= ex2(-dl);
            p[r] = valid ? ex2(s2[r] - m_run[r]) : 0.f;
            x[r] = p[r] * wv;
          }
          named_sync(gbar, 128);
          flip = true;
        }
        uint32_t X[kRows];
#pragma unroll
        for (int r = 0; r < kRows; ++r) {
          l_part[r] += p[r];
          X[r] = valid ? __float2uint_rn(x[r] * 16777216.f) : 0u;
        }
        // -- weights of the tile into P[xb] (xb = jt % 3), once the product
        // of tile jt - 3 has read it; the key group builds the value operand.
        const int xb = jt % kNVh;
        if (!__all_sync(0xffffffffu, mbar_wait(&vh_free[xb], ((jt / kNVh) & 1) ^ 1, A.wait_ns)) && lane == 0) fail();
        *reinterpret_cast<uint4*>(sm + Sm::kOffP + xb * 2048 + lrow * 16) = make_uint4(X[0], X[1], X[2], X[3]);
        if (lrow == 0) recs[(jt & 7) * 16 + 1] = flip ? 1u : 0u;
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&pv_ready[xb]);
        // The PV issuer closes the group's region before this tile's product;
        // fold it now (rare).
        if (flip && !fold(m_old)) {
          if (lane == 0) fail();
        }
      }
      cp_async_wait<0>();
      j = j0 + nt_tiles;
      // -------- segment end: the group's final region; its partial record
      // (v + s) * 2 + grp holds m, l and the rotated output sum.
      const int64_t rec = (sg.v + sg.s) * 2 + grp;
      if (nt_tiles > grp) {
        if (!stop && !fold(m_run)) {
          if (lane == 0) fail();
          stop = true;
        }
        if (!stop) {
#pragma unroll
          for (int r = 0; r < kRows; ++r) {
            const float x = warp_sum(l_part[r]);
            if (lane == 0) red[(8 + 4 * grp + q) * 16 + 8 + r] = x;
          }
        }
        named_sync(gbar, 128);
#pragma unroll
        for (int r = 0; r < kRows; ++r) {
          float* pr = a.part + (rec * kRows + r) * kRecFloats;
          pr[lrow] = acc[r] * v0;
          if (lrow == 0) {
            const float* rg = red + (8 + 4 * grp) * 16 + 8 + r;
            pr[kD] = m_run[r];
            pr[kD + 1] = rg[0] + rg[16] + rg[32] + rg[48];
          }
        }
      } else {
#pragma unroll
        for (int r = 0; r < kRows; ++r) {
          float* pr = a.part + (rec * kRows + r) * kRecFloats;
          pr[lrow] = 0.f;
          if (lrow == 0) {
            pr[kD] = -INFINITY;
            pr[kD + 1] = 0.f;
          }
        }
      }
      // ---------------- arrival; the stream's last segment merges. Both groups
      // pass the same barriers whether or not they stopped; the decision to
      // quit is taken once, after the first of them.
      __threadfence();
      named_sync(2, 256);
      if (u == 0) {
        merge_s[1] = *abort_s != 0 ? 1 : 0;
        const int64_t vf = vof(part, sg.s * part.Ts), vl = vof(part, (sg.s + 1) * part.Ts - 1);
        const int nseg = static_cast<int>(vl - vf + 1);
        const int old = atomicAdd(A.counters + sg.s, 1);
        const int last = old == nseg - 1;
        if (last) __threadfence();
        merge_s[0] = last ? 1 : 0;
        if (last) {
          reinterpret_cast<int64_t*>(red)[0] = vf;
          reinterpret_cast<int64_t*>(red)[1] = vl;
        }
      }
      named_sync(2, 256);
      if (merge_s[1]) break;
      if (merge_s[0]) {
        // Records of the stream (two per segment), merged online by group 0
        // (thread = coordinate, four records at a time with all loads in
        // flight); then out = Pi_V^T o_rot with the input coordinates split in
        // two (thread = output coordinate), partial sums through smem.
        const int64_t vf = reinterpret_cast<const int64_t*>(red)[0], vl = reinterpret_cast<const int64_t*>(red)[1];
        const int crd = u & 127, half = u >> 7;
        if (half == 0) {
          float M[kRows], L[kRows], O[kRows];
#pragma unroll
          for (int r = 0; r < kRows; ++r) {
            M[r] = -INFINITY;
            L[r] = 0.f;
            O[r] = 0.f;
          }
          const int64_t r0 = (vf + sg.s) * 2, r1 = (vl + sg.s) * 2 + 1;
          for (int64_t c0 = r0; c0 <= r1; c0 += 4) {
            float mk[4][kRows], lk[4][kRows], ok4[4][kRows];
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
#pragma unroll
              for (int r = 0; r < kRows; ++r) {
                const bool has = c0 + kk <= r1;
                const float* pr = a.part + ((c0 + kk) * kRows + r) * kRecFloats;
                mk[kk][r] = has ? __ldcg(pr + kD) : -INFINITY;
                lk[kk][r] = has ? __ldcg(pr + kD + 1) : 0.f;
                ok4[kk][r] = has ? __ldcg(pr + crd) : 0.f;
              }
#pragma unroll
            for (int r = 0; r < kRows; ++r) {
              float Mn = M[r];
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) Mn = fmaxf(Mn, mk[kk][r]);
              const float c = M[r] == -INFINITY ? 0.f : ex2(M[r] - Mn);
              L[r] *= c;
              O[r] *= c;
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                const float wgt = mk[kk][r] == -INFINITY ? 0.f : ex2(mk[kk][r] - Mn);
                L[r] = fmaf(lk[kk][r], wgt, L[r]);
                O[r] = fmaf(ok4[kk][r], wgt, O[r]);
              }
              M[r] = Mn;
            }
          }
#pragma unroll
          for (int r = 0; r < kRows; ++r) qx[r * kD + crd] = L[r] > 0.f ? O[r] / L[r] : 0.f;
        }
        named_sync(2, 256);
        const float* PV = a.PiV + int64_t(kv) * a.pi_stride;
        const int j_lo = half * 64;
        float o4[kRows] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 1
        for (int jb = 0; jb < 64; jb += 32) {
          float pv[32];
#pragma unroll
          for (int kk = 0; kk < 32; ++kk) pv[kk] = __ldg(PV + int64_t(j_lo + jb + kk) * kD + crd);
#pragma unroll
          for (int kk = 0; kk < 32; ++kk) {
#pragma unroll
            for (int r = 0; r < kRows; ++r) o4[r] = fmaf(pv[kk], qx[r * kD + j_lo + jb + kk], o4[r]);
          }
        }
        if (half == 1) {
#pragma unroll
          for (int r = 0; r < kRows; ++r) qr[r * kD + crd] = o4[r];
        }
        named_sync(2, 256);
        if (half == 0) {
#pragma unroll
          for (int r = 0; r < kRows; ++r) {
            const float v = o4[r] + qr[r * kD + crd];
            const int64_t oi = qrow(r) * kD + crd;
            if (a.out_dtype == 0) reinterpret_cast<float*>(a.out)[oi] = v;
            else reinterpret_cast<__nv_bfloat16*>(a.out)[oi] = __float2bfloat16_rn(v);
          }
          if (crd == 0) A.counters[sg.s] = 0;    // ready for the next call
        }
      }
      named_sync(2, 256);                         // qx / qr are the next prologue's again
    }
  }

  // ------------------------------------------------------------- teardown
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == kWScore) {
    tc_fence_after();
    __syncwarp();
    tmem_dealloc(tmem, kTmemCols);
  }
}

struct FusedPlan {
  int64_t T, Ts, streams;
  int V;
  size_t off_qprep, off_part, bytes;
};
// Partition and workspace of a call on `grid` CTAs: [arrival counters, one per
// stream | partial records, one per (virtual CTA, stream) pair index v + s].
FusedPlan fused_plan(const DecodeShape& s, int grid) {
  FusedPlan p{};
  p.streams = int64_t(s.batch) * s.hkv;
  p.Ts = (s.n_ctx + kTT - 1) / kTT;
  p.T = p.streams * p.Ts;
  const int64_t vmin = (p.T + kMaxSegTiles - 1) / kMaxSegTiles;
  // Every physical CTA gets the same number of virtual ones.
  p.V = static_cast<int>(((std::max<int64_t>(vmin, 1) + grid - 1) / grid) * grid);
  p.off_qprep = ((size_t(p.streams) * sizeof(int) + 255) / 256) * 256;
  p.off_part = p.off_qprep + size_t(p.streams) * kQPrepStride;
  p.bytes = p.off_part + size_t(p.V + p.streams) * 2 * kRows * kRecFloats * sizeof(float);
  return p;
}

int fused_grid(const DecodeShape& s, int sms) {
  const int64_t T = int64_t(s.batch) * s.hkv * ((s.n_ctx + kTT - 1) / kTT);
  return static_cast<int>(std::min<int64_t>(std::min(sms, kMaxGrid), T));
}

}  // namespace

bool tc_decode_supported(const DecodeArgs& v) {
  const DecodeShape& s = v.sh;
  if (s.d != kD || s.vbits != 3 || s.nq != 1 || s.hq != kRows * s.hkv) return false;
  if (s.kbits < 2 || s.kbits > 4) return false;
  // Bulk copies need 16-byte aligned sources: plane bases and stream offsets
  // (rows are multiples of 16 bytes); the prologue reads Pi_K and S rows as
  // float4.
  if (!aligned(v.kidx, 16) || !aligned(v.ksign, 16) || !aligned(v.vidx, 16)) return false;
  if (!aligned(v.PiK, 16) || !aligned(v.S, 16) || v.pi_stride % 4 != 0) return false;
  return true;
}

size_t tc_decode_workspace_bytes(const DecodeShape& s) {
  if (s.d != kD || s.vbits != 3 || s.nq != 1 || s.hq != kRows * s.hkv) return 0;
  return fused_plan(s, fused_grid(s, kMaxGrid)).bytes;     // covers every grid <= kMaxGrid
}

cudaError_t tc_decode_launch(const DecodeArgs& v, void* workspace, cudaStream_t st) {
  int dev = 0, sms = 148;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const int grid = fused_grid(v.sh, sms);
  const FusedPlan p = fused_plan(v.sh, grid);
  FusedArgs A{};
  A.v = v;
  A.T = p.T;
  A.Ts = p.Ts;
  A.V = p.V;
  A.counters = static_cast<int*>(workspace);
  A.wait_ns = pipeline_wait_ns();
  A.qprep = static_cast<unsigned char*>(workspace) + p.off_qprep;
  A.v.part = reinterpret_cast<float*>(static_cast<char*>(workspace) + p.off_part);
  e = cudaMemsetAsync(A.counters, 0, size_t(p.streams) * sizeof(int), st);
  if (e != cudaSuccess) return e;
  decode_qprep_kernel<<<static_cast<unsigned>(p.streams), 256, 0, st>>>(A);
  count_launch();
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  switch (v.sh.kbits) {
    case 2:
      e = cudaFuncSetAttribute(decode_fused_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, FSm<2>::kBytes);
      if (e == cudaSuccess) decode_fused_kernel<2><<<grid, kThreads, FSm<2>::kBytes, st>>>(A);
      break;
    case 3:
      e = cudaFuncSetAttribute(decode_fused_kernel<3>, cudaFuncAttributeMaxDynamicSharedMemorySize, FSm<3>::kBytes);
      if (e == cudaSuccess) decode_fused_kernel<3><<<grid, kThreads, FSm<3>::kBytes, st>>>(A);
      break;
    default:
      e = cudaFuncSetAttribute(decode_fused_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, FSm<4>::kBytes);
      if (e == cudaSuccess) decode_fused_kernel<4><<<grid, kThreads, FSm<4>::kBytes, st>>>(A);
      break;
  }
  if (e != cudaSuccess) return e;
  count_launch();
  return cudaGetLastError();
}

}  // namespace tq
