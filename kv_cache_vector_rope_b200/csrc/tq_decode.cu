// tq_decode_attention: softmax attention computed directly over the packed
// K/V planes.
//
// Sources: gist.science "TurboESM ..." section 2E (one fused kernel: unpack
// 3-bit codes, QJL correction, inverse rotation Pi^T, online softmax; no
// dequantised tensor in memory) and 7minutos.es "KV cache ... TurboQuant"
// Etapa 2 (sign bits enter through S^T scaled by sqrt(pi/2)/d and ||r||).
//
// Three launches on the caller's stream:
//   1. prologue  q_rot = Pi_K RoPE(q), s = S q_rot for every query row.
//   2. main      one CTA per (KV stream, query-row block, context split).
//                Scores use per-CTA shared-memory tables
//                  Tk[i][c][r] = q_rot[r][i] * cK[c]        (code lookups)
//                  Ts[i/4][m][r] = sum over 4 coords of +-s (sign nibbles)
//                so a key costs one table read per coordinate and one per 4
//                sign bits; V is accumulated in rotated coordinates with an
//                online softmax; each CTA leaves (m, l, acc) for its split.
//   3. combine   merges the splits and applies Pi_V^T once per query row.
// Shapes the fused tensor-core kernel takes (d = 128, four query heads per KV
// head, one query each, 3-bit values; tq_decode_tc.cu) go there instead;
// TQ_DECODE_PATH=v1 or v2 keeps them on these kernels (v2: the table kernel of
// tq_decode_v2.cuh, v1: the general one).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "tq_device.cuh"
#include "tq_internal.h"
#include "tq_decode_tc.h"

namespace tq {
namespace {

using namespace dev;

constexpr int kT = 128;              // tokens per tile = threads of the main kernel
constexpr int kTargetCtas = 1024;    // split heuristic target (shape-only, device independent)
constexpr int kMaxRows = 8;          // query rows per main-kernel CTA

int pick_rows(int group_rows) {
  for (int r = kMaxRows; r >= 1; r >>= 1)
    if (group_rows % r == 0) return r;
  return 1;
}

DecodeShape make_shape(const tq_layout* L, int batch, int hq, int hkv, int nq, int64_t n_ctx, int64_t ctx_stride) {
  DecodeShape s{};
  s.d = L->d;
  s.kbits = L->key_bits;
  s.vbits = L->value_bits;
  s.batch = batch;
  s.hq = hq;
  s.hkv = hkv;
  s.nq = nq;
  s.n_ctx = n_ctx;
  s.ctx_stride = ctx_stride ? ctx_stride : n_ctx;
  const int group_rows = (hq / hkv) * nq;
  s.rows_per_cta = pick_rows(group_rows);
  s.row_blocks = group_rows / s.rows_per_cta;
  const int64_t units = int64_t(batch) * hkv * s.row_blocks;
  const int64_t tiles = (n_ctx + kT - 1) / kT;
  int64_t splits = std::max<int64_t>(1, (kTargetCtas + units - 1) / units);
  splits = std::min(splits, tiles);
  const int64_t per = (tiles + splits - 1) / splits;
  s.chunk = per * kT;
  s.n_splits = static_cast<int>((n_ctx + s.chunk - 1) / s.chunk);
  s.n_parts = s.n_splits;
  s.n_rows = int64_t(batch) * hq * nq;
  return s;
}

size_t shape_workspace_bytes(const DecodeShape& s) {
  const size_t qs = size_t(s.n_rows) * 2 * s.d * sizeof(float);
  const size_t part = size_t(s.n_rows) * s.n_splits * (s.d + 2) * sizeof(float);
  return ((qs + 255) / 256) * 256 + part;
}

// Query row index -> (b, h, n).
__device__ __forceinline__ void row_coords(const DecodeShape& s, int64_t row, int& b, int& h, int& n) {
  n = static_cast<int>(row % s.nq);
  const int64_t bh = row / s.nq;
  h = static_cast<int>(bh % s.hq);
  b = static_cast<int>(bh / s.hq);
}

// ---------------------------------------------------------------------------
// Row blocks of the prologue and the combine: up to 16 query rows that share
// one rotation (all rows when Pi is shared, else the G*nq rows of one
// (batch, KV head) stream). Each CTA stages the d x d matrix once in shared
// memory (row pitch d+1: conflict-free reads along either index) and applies
// it to its rows; thread (i, group) owns coordinate i of RPG rows.
// ---------------------------------------------------------------------------
constexpr int kBlkRows = 16;
constexpr int kBlkThreads = 256;
constexpr int kCombChunk = 64;       // partial records whose weights are staged at a time

struct RowBlocks {
  int rows_per_group, blocks_per_group, n_blocks;
};

RowBlocks row_blocks(const DecodeShape& s, int64_t pi_stride) {
  RowBlocks r{};
  r.rows_per_group = pi_stride == 0 ? static_cast<int>(s.n_rows) : (s.hq / s.hkv) * s.nq;
  r.blocks_per_group = (r.rows_per_group + kBlkRows - 1) / kBlkRows;
  r.n_blocks = static_cast<int>(s.n_rows / r.rows_per_group) * r.blocks_per_group;
  return r;
}

// Row groups per CTA: floor(256 / d) capped at 4, a power of two.
inline int row_groups(int d) { return d <= 64 ? 4 : (d <= 128 ? 2 : 1); }
inline size_t blk_smem_bytes(int d) { return sizeof(float) * (size_t(d) * (d + 1) + 2 * size_t(d) * kBlkRows); }

// Stages the d x d row-major matrix M into Ms (pitch d+1): every thread first
// loads its float4s of the matrix (independent, coalesced loads), then stores
// them.
__device__ __forceinline__ void stage_matrix(float* Ms, const float* __restrict__ M, int d) {
  const int n4 = d * d / 4, q4 = d / 4;
  constexpr int kMaxPer = (256 * 256 / 4) / kBlkThreads;
  float4 v[8];
  for (int e0 = 0; e0 < n4; e0 += 8 * kBlkThreads) {
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int e = e0 + threadIdx.x + u * kBlkThreads;
      if (e < n4) v[u] = __ldg(reinterpret_cast<const float4*>(M) + e);
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int e = e0 + threadIdx.x + u * kBlkThreads;
      if (e < n4) {
        float* dst = Ms + (e / q4) * (d + 1) + 4 * (e % q4);
        dst[0] = v[u].x;
        dst[1] = v[u].y;
        dst[2] = v[u].z;
        dst[3] = v[u].w;
      }
    }
  }
  (void)kMaxPer;
}

// out[r][i] = sum_j Ms[i][j] xs[j][r] (TRANS = false) or sum_j Ms[j][i] xs[j][r]
// (TRANS = true) for the RPG rows of this thread's group; xs is j-major
// [d][16]. Returns false for threads without a coordinate.
template <int RPG, bool TRANS>
__device__ __forceinline__ bool blk_matvec(const float* Ms, const float* xs, int d, float (&acc)[RPG], int& i, int& r0) {
  const int t = threadIdx.x;
  const int groups = kBlkRows / RPG;
  if (t >= groups * d) return false;
  i = t % d;
  r0 = (t / d) * RPG;
#pragma unroll
  for (int u = 0; u < RPG; ++u) acc[u] = 0.f;
  const int pitch = d + 1;
  for (int j = 0; j < d; ++j) {
    const float m = TRANS ? Ms[j * pitch + i] : Ms[i * pitch + j];
    const float4* x4 = reinterpret_cast<const float4*>(xs + j * kBlkRows + r0);
#pragma unroll
    for (int u4 = 0; u4 < RPG / 4; ++u4) {
      const float4 x = x4[u4];
      acc[4 * u4 + 0] = fmaf(m, x.x, acc[4 * u4 + 0]);
      acc[4 * u4 + 1] = fmaf(m, x.y, acc[4 * u4 + 1]);
      acc[4 * u4 + 2] = fmaf(m, x.z, acc[4 * u4 + 2]);
      acc[4 * u4 + 3] = fmaf(m, x.w, acc[4 * u4 + 3]);
    }
  }
  return true;
}

// ---------------------------------------------------------------------------
// 1. Prologue: q_rot = Pi_K[kv] RoPE(q), s = S q_rot for every query row.
// ---------------------------------------------------------------------------
template <int RPG>
__global__ void __launch_bounds__(kBlkThreads) decode_prologue(DecodeArgs a, RowBlocks rb) {
  extern __shared__ __align__(16) float blk_smem[];
  const DecodeShape& s = a.sh;
  const int d = s.d;
  float* Ms = blk_smem;                       // [d][d+1]
  float* xs = Ms + d * (d + 1);               // [d][16] RoPE'd queries
  float* ys = xs + d * kBlkRows;              // [d][16] q_rot
  const int g = blockIdx.x / rb.blocks_per_group, sub = blockIdx.x % rb.blocks_per_group;
  const int64_t row0 = int64_t(g) * rb.rows_per_group + sub * kBlkRows;
  const int cnt = min(kBlkRows, rb.rows_per_group - sub * kBlkRows);
  const int kv = a.pi_stride ? g % s.hkv : 0;
  stage_matrix(Ms, a.PiK + kv * a.pi_stride, d);
  const bool rope = a.q_pos != nullptr && a.rope_base > 0.0;
  for (int e = threadIdx.x; e < kBlkRows * (d / 2); e += kBlkThreads) {
    const int r = e / (d / 2), i = e % (d / 2);
    float x0 = 0.f, x1 = 0.f;
    if (r < cnt) {
      const int64_t row = row0 + r;
      x0 = load_elem(a.q, a.q_dtype, row * d + i);
      x1 = load_elem(a.q, a.q_dtype, row * d + i + d / 2);
      if (rope) {
        int b, h, n;
        row_coords(s, row, b, h, n);
        const int pos = a.q_pos[int64_t(b) * s.nq + n];
        if (pos < 0 && a.d_status) atomicOr(a.d_status, TQ_DEV_BAD_POSITION);
        double sn, cs;
        sincos(rope_angle(pos, i, d, a.rope_base), &sn, &cs);
        const double r0 = double(x0) * cs - double(x1) * sn, r1 = double(x0) * sn + double(x1) * cs;
        x0 = static_cast<float>(r0);
        x1 = static_cast<float>(r1);
      }
    }
    xs[i * kBlkRows + r] = x0;
    xs[(i + d / 2) * kBlkRows + r] = x1;
  }
  __syncthreads();
  float acc[RPG];
  int i, r0;
  if (blk_matvec<RPG, false>(Ms, xs, d, acc, i, r0)) {
#pragma unroll
    for (int u = 0; u < RPG; ++u) {
      ys[i * kBlkRows + r0 + u] = acc[u];
      if (r0 + u < cnt) a.qs[(row0 + r0 + u) * 2 * d + i] = acc[u];
    }
  }
  __syncthreads();
  stage_matrix(Ms, a.S, d);
  __syncthreads();
  if (blk_matvec<RPG, false>(Ms, ys, d, acc, i, r0)) {
#pragma unroll
    for (int u = 0; u < RPG; ++u)
      if (r0 + u < cnt) a.qs[(row0 + r0 + u) * 2 * d + d + i] = acc[u];
  }
}

// Cooperative byte copy global -> shared with 16-byte vectors when possible.
__device__ __forceinline__ void stage(void* dst, const void* src, int64_t bytes) {
  const bool vec = ((reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst) | bytes) & 15) == 0;
  if (vec) {
    const uint4* s4 = reinterpret_cast<const uint4*>(src);
    uint4* d4 = reinterpret_cast<uint4*>(dst);
    for (int64_t i = threadIdx.x; i < bytes / 16; i += blockDim.x) d4[i] = __ldg(s4 + i);
  } else {
    const uint8_t* s1 = reinterpret_cast<const uint8_t*>(src);
    uint8_t* d1 = reinterpret_cast<uint8_t*>(dst);
    for (int64_t i = threadIdx.x; i < bytes; i += blockDim.x) d1[i] = s1[i];
  }
}

__device__ __forceinline__ uint32_t group_word(const uint8_t* row, int g, int bits) {
  const uint8_t* p = row + g * bits;
  uint32_t w = 0;
  for (int b = 0; b < bits; ++b) w |= static_cast<uint32_t>(p[b]) << (8 * b);
  return w;
}

// ---------------------------------------------------------------------------
// 2. Main split-KV kernel.
// ---------------------------------------------------------------------------
template <int D, int R>
struct MainSmem {
  static constexpr int kSW = (D + 31) / 32;
  float sc[kT][R];           // scores of the tile
  float w[kT][R];            // exp(score - m) * ||v||
  float knorm[kT], krn[kT], vnorm[kT];
  uint32_t ksign[kT][kSW];
  float red[kT / kWarp][R];
  float m[R], l[R], corr[R];
  float cV[16];
  // followed by: Tk[D][nck][R], Ts[D/4][16][R], kidx[kT*rbk], vidx[kT*rbv]
};

template <int D, int R>
__global__ void __launch_bounds__(kT) decode_main(DecodeArgs a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  using Sm = MainSmem<D, R>;
  Sm& s = *reinterpret_cast<Sm*>(smem_raw);
  const DecodeShape& sh = a.sh;
  const int nck = 1 << sh.kbits, ncv = 1 << sh.vbits;
  const int rbk = D * sh.kbits / 8, rbv = D * sh.vbits / 8;
  float* Tk = reinterpret_cast<float*>(smem_raw + ((sizeof(Sm) + 15) / 16) * 16);
  float* Ts = Tk + D * nck * R;
  uint8_t* kidx = reinterpret_cast<uint8_t*>(Ts + (D / 4) * 16 * R);
  uint8_t* vidx = kidx + ((kT * rbk + 15) / 16) * 16;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int split = blockIdx.x;
  const int64_t unit = blockIdx.y;                      // (b, kv, row block)
  const int rb = static_cast<int>(unit % sh.row_blocks);
  const int64_t bkv = unit / sh.row_blocks;             // b*hkv + kv
  const int G = sh.hq / sh.hkv;
  const int kv = static_cast<int>(bkv % sh.hkv);
  const int b = static_cast<int>(bkv / sh.hkv);
  // Query row r of this CTA: group-local index rr = rb*R + r -> head kv*G + rr/nq, query rr%nq.
  auto qrow = [&](int r) -> int64_t {
    const int rr = rb * R + r;
    const int h = kv * G + rr / sh.nq;
    return (int64_t(b) * sh.hq + h) * sh.nq + rr % sh.nq;
  };

  // Tables.
  if (tid < ncv) s.cV[tid] = a.cV[tid];
  for (int e = tid; e < D * nck * R; e += kT) {
    const int r = e % R, c = (e / R) % nck, i = e / (R * nck);
    Tk[e] = a.qs[qrow(r) * 2 * D + i] * __ldg(a.cK + c);
  }
  for (int e = tid; e < (D / 4) * 16 * R; e += kT) {
    const int r = e % R, m = (e / R) % 16, nib = e / (R * 16);
    const float* sv = a.qs + qrow(r) * 2 * D + D + 4 * nib;
    float acc = 0.f;
#pragma unroll
    for (int q = 0; q < 4; ++q) acc += ((m >> q) & 1) ? sv[q] : -sv[q];
    Ts[e] = acc;
  }
  if (tid < R) {
    s.m[tid] = -INFINITY;
    s.l[tid] = 0.f;
  }
  float acc[(D + kT - 1) / kT][R];
#pragma unroll
  for (int c = 0; c < (D + kT - 1) / kT; ++c)
#pragma unroll
    for (int r = 0; r < R; ++r) acc[c][r] = 0.f;

  const float alpha = static_cast<float>(kSqrtHalfPi / D);
  const int64_t t_begin = int64_t(split) * sh.chunk;
  const int64_t t_end = (t_begin + sh.chunk < sh.n_ctx) ? t_begin + sh.chunk : sh.n_ctx;
  const int64_t row0 = bkv * sh.ctx_stride;

  for (int64_t t0 = t_begin; t0 < t_end; t0 += kT) {
    const int nt = static_cast<int>((t_end - t0 < kT) ? t_end - t0 : kT);
    __syncthreads();
    stage(kidx, a.kidx + (row0 + t0) * rbk, int64_t(nt) * rbk);
    stage(vidx, a.vidx + (row0 + t0) * rbv, int64_t(nt) * rbv);
    stage(&s.ksign[0][0], a.ksign + (row0 + t0) * Sm::kSW, int64_t(nt) * Sm::kSW * 4);
    if (tid < nt) {
      s.knorm[tid] = __ldg(a.knorm + row0 + t0 + tid);
      s.krn[tid] = __ldg(a.krnorm + row0 + t0 + tid);
      s.vnorm[tid] = __ldg(a.vnorm + row0 + t0 + tid);
    }
    __syncthreads();

    // Scores: thread = token.
    float score[R];
    if (tid < nt) {
      float ck[R], cs[R];
#pragma unroll
      for (int r = 0; r < R; ++r) ck[r] = cs[r] = 0.f;
      const uint8_t* row = kidx + tid * rbk;
      for (int g = 0; g < D / 8; ++g) {
        const uint32_t word = group_word(row, g, sh.kbits);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int c = (word >> (sh.kbits * j)) & (nck - 1);
          const float* e = Tk + ((8 * g + j) * nck + c) * R;
#pragma unroll
          for (int r = 0; r < R; ++r) ck[r] += e[r];
        }
      }
      for (int nib = 0; nib < D / 4; ++nib) {
        const int m = (s.ksign[tid][nib >> 3] >> (4 * (nib & 7))) & 15;
        const float* e = Ts + (nib * 16 + m) * R;
#pragma unroll
        for (int r = 0; r < R; ++r) cs[r] += e[r];
      }
      const float kn = s.knorm[tid], rn = s.krn[tid];
#pragma unroll
      for (int r = 0; r < R; ++r) score[r] = a.scale * (kn * ck[r] + alpha * rn * cs[r]);
    } else {
#pragma unroll
      for (int r = 0; r < R; ++r) score[r] = -INFINITY;
    }
#pragma unroll
    for (int r = 0; r < R; ++r) s.sc[tid][r] = score[r];
    if (a.scores_out && tid < nt) {
#pragma unroll
      for (int r = 0; r < R; ++r) a.scores_out[qrow(r) * sh.n_ctx + t0 + tid] = score[r];
    }
    // Tile max per row.
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const float mx = warp_max(score[r]);
      if (lane == 0) s.red[warp][r] = mx;
    }
    __syncthreads();
    if (tid < R) {
      float mx = s.red[0][tid];
      for (int w2 = 1; w2 < kT / kWarp; ++w2) mx = fmaxf(mx, s.red[w2][tid]);
      const float m_new = fmaxf(s.m[tid], mx);
      s.corr[tid] = (s.m[tid] == -INFINITY) ? 0.f : expf(s.m[tid] - m_new);
      s.m[tid] = m_new;
    }
    __syncthreads();
    float psum[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const float p = (tid < nt) ? expf(score[r] - s.m[r]) : 0.f;
      s.w[tid][r] = p * ((tid < nt) ? s.vnorm[tid] : 0.f);
      psum[r] = warp_sum(p);
    }
#pragma unroll
    for (int r = 0; r < R; ++r)
      if (lane == 0) s.red[warp][r] = psum[r];
    __syncthreads();
    if (tid < R) {
      float tot = 0.f;
      for (int w2 = 0; w2 < kT / kWarp; ++w2) tot += s.red[w2][tid];
      s.l[tid] = s.l[tid] * s.corr[tid] + tot;
    }
    // V: thread = coordinate.
#pragma unroll
    for (int c = 0; c < (D + kT - 1) / kT; ++c) {
      const int i = tid + c * kT;
      if (i < D) {
#pragma unroll
        for (int r = 0; r < R; ++r) acc[c][r] *= s.corr[r];
        for (int t = 0; t < nt; ++t) {
          const float cv = s.cV[get_code(vidx + t * rbv, i, sh.vbits)];
#pragma unroll
          for (int r = 0; r < R; ++r) acc[c][r] = fmaf(s.w[t][r], cv, acc[c][r]);
        }
      }
    }
  }
  __syncthreads();
  // Partials.
#pragma unroll
  for (int c = 0; c < (D + kT - 1) / kT; ++c) {
    const int i = tid + c * kT;
    if (i < D) {
#pragma unroll
      for (int r = 0; r < R; ++r) a.part[(qrow(r) * sh.n_parts + split) * (D + 2) + i] = acc[c][r];
    }
  }
  if (tid < R) {
    float* p = a.part + (qrow(tid) * sh.n_parts + split) * (D + 2);
    p[D] = s.m[tid];
    p[D + 1] = s.l[tid];
  }
}

// ---------------------------------------------------------------------------
// 3. Combine the splits and turn back by Pi_V^T (a block of query rows per CTA).
// ---------------------------------------------------------------------------
template <int RPG>
__global__ void __launch_bounds__(kBlkThreads) decode_combine(DecodeArgs a, RowBlocks rb) {
  extern __shared__ __align__(16) float blk_smem[];
  const DecodeShape& s = a.sh;
  const int d = s.d, ns = s.n_parts;
  float* Ms = blk_smem;                       // [d][d+1] Pi_V
  float* os = Ms + d * (d + 1);               // [d][16] merged rotated outputs
  float* wl = os + d * kBlkRows;              // [16] 1 / L per row; [16] max per row; [16][64] weights
  const int g = blockIdx.x / rb.blocks_per_group, sub = blockIdx.x % rb.blocks_per_group;
  const int64_t row0 = int64_t(g) * rb.rows_per_group + sub * kBlkRows;
  const int cnt = min(kBlkRows, rb.rows_per_group - sub * kBlkRows);
  const int kv = a.pi_stride ? g % s.hkv : 0;
  stage_matrix(Ms, a.PiV + kv * a.pi_stride, d);
  float* wk = wl + 2 * kBlkRows;               // [16][kCombChunk] record weights
  // Row maxima and softmax denominators: warp w handles rows w and w + 8;
  // with at most kCombChunk records the record weights come out of the same
  // pass (lane k holds records k and k + 32).
  const bool one_pass = ns <= kCombChunk;
  {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int r = warp; r < kBlkRows; r += kBlkThreads / 32) {
      float M = -INFINITY, L = 0.f;
      if (r < cnt) {
        const float* part = a.part + (row0 + r) * ns * (d + 2);
        if (one_pass) {
          const bool h0 = lane < ns, h1 = lane + 32 < ns;
          const float m0 = h0 ? part[lane * (d + 2) + d] : -INFINITY;
          const float l0 = h0 ? part[lane * (d + 2) + d + 1] : 0.f;
          const float m1 = h1 ? part[(lane + 32) * (d + 2) + d] : -INFINITY;
          const float l1 = h1 ? part[(lane + 32) * (d + 2) + d + 1] : 0.f;
          M = warp_max(fmaxf(m0, m1));
          const float w0 = m0 > -INFINITY ? __expf(m0 - M) : 0.f;
          const float w1 = m1 > -INFINITY ? __expf(m1 - M) : 0.f;
          L = warp_sum(w0 * l0 + w1 * l1);
          wk[r * kCombChunk + lane] = w0;
          wk[r * kCombChunk + lane + 32] = w1;
        } else {
          for (int k = lane; k < ns; k += 32) M = fmaxf(M, part[k * (d + 2) + d]);
          M = warp_max(M);
          for (int k = lane; k < ns; k += 32) {
            const float mk = part[k * (d + 2) + d];
            if (mk > -INFINITY) L += __expf(mk - M) * part[k * (d + 2) + d + 1];
          }
          L = warp_sum(L);
        }
      } else if (one_pass) {
        wk[r * kCombChunk + lane] = 0.f;
        wk[r * kCombChunk + lane + 32] = 0.f;
      }
      if (lane == 0) {
        wl[r] = (r < cnt && L > 0.f) ? 1.f / L : 0.f;
        wl[kBlkRows + r] = M;
      }
    }
  }
  __syncthreads();
  // Merged rotated output o[r][i] = sum_k e^(m_k - M) acc_k[i] / L, with the
  // weights of kCombChunk records at a time staged in shared memory so the
  // record loads of a thread are independent (and coalesced over i).
  for (int e = threadIdx.x; e < kBlkRows * d; e += kBlkThreads) os[(e % d) * kBlkRows + e / d] = 0.f;
  for (int k0 = 0; k0 < ns; k0 += kCombChunk) {
    const int kn = min(kCombChunk, ns - k0);
    __syncthreads();
    if (!one_pass)
    for (int e = threadIdx.x; e < kBlkRows * kCombChunk; e += kBlkThreads) {
      const int r = e / kCombChunk, kk = e % kCombChunk;
      float w = 0.f;
      if (r < cnt && kk < kn) {
        const float mk = a.part[((row0 + r) * ns + k0 + kk) * (d + 2) + d];
        if (mk > -INFINITY) w = __expf(mk - wl[kBlkRows + r]);
      }
      wk[e] = w;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < kBlkRows * d; e += kBlkThreads) {
      const int r = e / d, i = e % d;
      if (r >= cnt) continue;
      const float* rec = a.part + ((row0 + r) * ns + k0) * (d + 2) + i;
      const float* w = wk + r * kCombChunk;
      float o0 = 0.f, o1 = 0.f;
      int kk = 0;
#pragma unroll 4
      for (; kk + 1 < kn; kk += 2) {
        o0 = fmaf(w[kk], rec[kk * (d + 2)], o0);
        o1 = fmaf(w[kk + 1], rec[(kk + 1) * (d + 2)], o1);
      }
      if (kk < kn) o0 = fmaf(w[kk], rec[kk * (d + 2)], o0);
      os[i * kBlkRows + r] += o0 + o1;
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < kBlkRows * d; e += kBlkThreads) {
    const int r = e / d, i = e % d;
    os[i * kBlkRows + r] *= wl[r];
  }
  __syncthreads();
  float acc[RPG];
  int j, r0;
  if (blk_matvec<RPG, true>(Ms, os, d, acc, j, r0)) {
#pragma unroll
    for (int u = 0; u < RPG; ++u) {
      if (r0 + u >= cnt) continue;
      const int64_t row = row0 + r0 + u;
      if (a.out_dtype == 0)
        reinterpret_cast<float*>(a.out)[row * d + j] = acc[u];
      else
        reinterpret_cast<__nv_bfloat16*>(a.out)[row * d + j] = __float2bfloat16(acc[u]);
    }
  }
}

// ---------------------------------------------------------------------------
// Few query rows (the GQA decode shape): one CTA of d threads per row, the
// matrices read straight from L2 (no staging), so the prologue and the
// combine spread over many SMs with every load coalesced.
// ---------------------------------------------------------------------------
constexpr int kRowWarpMaxRows = 512;         // above this, the row-block kernels

// The row's Pi (shared, or the row's KV head's).
__device__ __forceinline__ int row_kv(const DecodeArgs& a, int64_t row) {
  if (!a.pi_stride) return 0;
  const int64_t rows_per_group = int64_t(a.sh.hq / a.sh.hkv) * a.sh.nq;
  return static_cast<int>((row / rows_per_group) % a.sh.hkv);
}

// y[i] = sum_j M[i][j] v[j] for the D/32 rows i = 32 w + o handled by warp w:
// lane l reads M[i][G l .. G l + G) (one coalesced row read per i) and the
// warp sums the products. v in shared memory; y written to ys (shared) and out.
template <int D>
__device__ __forceinline__ void row_matvec_warps(const float* __restrict__ M, const float* v, float* ys,
                                                 float* __restrict__ out) {
  constexpr int G = D / 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float x[G];
#pragma unroll
  for (int c = 0; c < G; ++c) x[c] = v[G * lane + c];
  constexpr int kRowsPerWarp = D / (D / 32);    // 32 rows per warp (D/32 warps)
#pragma unroll 8
  for (int o = 0; o < kRowsPerWarp; ++o) {
    const int i = warp * kRowsPerWarp + o;
    float p;
    if constexpr (G == 4) {
      const float4 m = __ldg(reinterpret_cast<const float4*>(M + i * D) + lane);
      p = fmaf(m.x, x[0], fmaf(m.y, x[1], fmaf(m.z, x[2], m.w * x[3])));
    } else {
      const float2 m = __ldg(reinterpret_cast<const float2*>(M + i * D) + lane);
      p = fmaf(m.x, x[0], m.y * x[1]);
    }
    p = warp_sum(p);
    if (lane == 0) {
      if (ys) ys[i] = p;
      out[i] = p;
    }
  }
}

template <int D>
__global__ void __launch_bounds__(D) decode_prologue_rows(DecodeArgs a) {
  __shared__ __align__(16) float xs[D], ys[D];
  const DecodeShape& s = a.sh;
  const int64_t row = blockIdx.x;
  const int i = threadIdx.x;
  const int kv = row_kv(a, row);
  // RoPE pairs (i, i + D/2).
  if (i < D / 2) {
    float x0 = load_elem(a.q, a.q_dtype, row * D + i);
    float x1 = load_elem(a.q, a.q_dtype, row * D + i + D / 2);
    if (a.q_pos != nullptr && a.rope_base > 0.0) {
      int b, h, n;
      row_coords(s, row, b, h, n);
      const int pos = a.q_pos[int64_t(b) * s.nq + n];
      if (pos < 0 && a.d_status && i == 0) atomicOr(a.d_status, TQ_DEV_BAD_POSITION);
      double sn, cs;
      sincos(rope_angle(pos, i, D, a.rope_base), &sn, &cs);
      const double r0 = double(x0) * cs - double(x1) * sn, r1 = double(x0) * sn + double(x1) * cs;
      x0 = static_cast<float>(r0);
      x1 = static_cast<float>(r1);
    }
    xs[i] = x0;
    xs[i + D / 2] = x1;
  }
  __syncthreads();
  row_matvec_warps<D>(a.PiK + int64_t(kv) * a.pi_stride, xs, ys, a.qs + row * 2 * D);
  __syncthreads();
  row_matvec_warps<D>(a.S, ys, nullptr, a.qs + row * 2 * D + D);
}

template <int D>
__global__ void __launch_bounds__(D) decode_combine_rows(DecodeArgs a) {
  __shared__ __align__(16) float os[D];
  __shared__ float wk[64];
  __shared__ float inv_l_s;
  const DecodeShape& s = a.sh;
  const int ns = s.n_parts;
  const int64_t row = blockIdx.x;
  const int i = threadIdx.x, warp = i >> 5, lane = i & 31;
  const int kv = row_kv(a, row);
  const float* part = a.part + row * ns * (D + 2);
  // Row maximum and softmax denominator (warp 0); the record weights go to
  // shared memory when they fit (else every thread forms them itself).
  if (warp == 0) {
    float M = -INFINITY;
    for (int k = lane; k < ns; k += 32) M = fmaxf(M, part[k * (D + 2) + D]);
    M = warp_max(M);
    float L = 0.f;
    for (int k = lane; k < ns; k += 32) {
      const float mk = part[k * (D + 2) + D];
      const float w = mk > -INFINITY ? __expf(mk - M) : 0.f;
      if (k < 64) wk[k] = w;
      L += w * part[k * (D + 2) + D + 1];
    }
    L = warp_sum(L);
    if (lane == 0) inv_l_s = L > 0.f ? 1.f / L : 0.f;
    if (lane == 0 && ns > 64) wk[0] = M;          // the reference for the slow path
  }
  __syncthreads();
  float o = 0.f;
  if (ns <= 64) {
#pragma unroll 8
    for (int k = 0; k < ns; ++k) o = fmaf(wk[k], part[k * (D + 2) + i], o);
  } else {
    const float M = wk[0];
    for (int k = 0; k < ns; ++k) {
      const float mk = part[k * (D + 2) + D];
      if (mk > -INFINITY) o = fmaf(__expf(mk - M), part[k * (D + 2) + i], o);
    }
  }
  os[i] = o * inv_l_s;
  __syncthreads();
  // out[j] = sum_i Pi_V[i][j] o[i], thread j (coalesced reads of row i).
  const float* PiV = a.PiV + int64_t(kv) * a.pi_stride;
  float acc = 0.f;
#pragma unroll 16
  for (int r = 0; r < D; ++r) acc = fmaf(__ldg(PiV + r * D + i), os[r], acc);
  const int64_t at = row * D + i;
  if (a.out_dtype == 0)
    reinterpret_cast<float*>(a.out)[at] = acc;
  else
    reinterpret_cast<__nv_bfloat16*>(a.out)[at] = __float2bfloat16(acc);
}

template <bool COMBINE>
cudaError_t launch_rows(const DecodeArgs& a, cudaStream_t st) {
  const unsigned grid = static_cast<unsigned>(a.sh.n_rows);
  if (a.sh.d == 128) {
    if (COMBINE) decode_combine_rows<128><<<grid, 128, 0, st>>>(a);
    else decode_prologue_rows<128><<<grid, 128, 0, st>>>(a);
  } else {
    if (COMBINE) decode_combine_rows<64><<<grid, 64, 0, st>>>(a);
    else decode_prologue_rows<64><<<grid, 64, 0, st>>>(a);
  }
  count_launch();
  return cudaGetLastError();
}

template <bool COMBINE>
cudaError_t launch_blk(const DecodeArgs& a, cudaStream_t st) {
  // Few rows of d = 64 or 128 (16-byte aligned matrices): one warp per row.
  const bool aligned_mats = ((reinterpret_cast<uintptr_t>(a.PiK) | reinterpret_cast<uintptr_t>(a.PiV) |
                              reinterpret_cast<uintptr_t>(a.S) | (a.pi_stride * sizeof(float))) & 15) == 0;
  if ((a.sh.d == 64 || a.sh.d == 128) && a.sh.n_rows <= kRowWarpMaxRows && aligned_mats)
    return launch_rows<COMBINE>(a, st);
  const RowBlocks rb = row_blocks(a.sh, a.pi_stride);
  const size_t smem = blk_smem_bytes(a.sh.d) + (COMBINE ? (2 + kCombChunk) * kBlkRows * sizeof(float) : 0);
  const int rg = row_groups(a.sh.d);
  auto kern = COMBINE ? (rg == 4 ? decode_combine<4> : rg == 2 ? decode_combine<8> : decode_combine<16>)
                      : (rg == 4 ? decode_prologue<4> : rg == 2 ? decode_prologue<8> : decode_prologue<16>);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  kern<<<static_cast<unsigned>(rb.n_blocks), kBlkThreads, smem, st>>>(a, rb);
  count_launch();
  return cudaGetLastError();
}

}  // namespace
}  // namespace tq

#include "tq_decode_v2.cuh"

namespace tq {
namespace {

template <int D, int R, int KB>
cudaError_t launch_v2(const DecodeArgs& a, cudaStream_t st) {
  using Sm = V2Smem<D, R, KB>;
  cudaError_t e = cudaFuncSetAttribute(decode_main_v2<D, R, KB>, cudaFuncAttributeMaxDynamicSharedMemorySize, Sm::kBytes);
  if (e != cudaSuccess) return e;
  dim3 grid(a.sh.n_splits, static_cast<unsigned>(int64_t(a.sh.batch) * a.sh.hkv * a.sh.row_blocks));
  decode_main_v2<D, R, KB><<<grid, kT2, Sm::kBytes, st>>>(a);
  count_launch();
  return cudaGetLastError();
}

// Version-2 kernel when it applies: d 64/128, 4 or 8 query rows per CTA,
// 3-bit values. Returns false to fall back to the general kernel.
template <int D>
bool try_v2(const DecodeArgs& a, cudaStream_t st, cudaError_t& e) {
  if (a.sh.vbits != 3 || !(a.sh.rows_per_cta == 4 || a.sh.rows_per_cta == 8)) return false;
  const bool r4 = a.sh.rows_per_cta == 4;
  switch (a.sh.kbits) {
    case 2: e = r4 ? launch_v2<D, 4, 2>(a, st) : launch_v2<D, 8, 2>(a, st); return true;
    case 3: e = r4 ? launch_v2<D, 4, 3>(a, st) : launch_v2<D, 8, 3>(a, st); return true;
    case 4: e = r4 ? launch_v2<D, 4, 4>(a, st) : launch_v2<D, 8, 4>(a, st); return true;
    default: return false;
  }
}

template <int D, int R>
cudaError_t launch_main(const DecodeArgs& a, cudaStream_t st) {
  using Sm = MainSmem<D, R>;
  const int nck = 1 << a.sh.kbits;
  const int rbk = D * a.sh.kbits / 8, rbv = D * a.sh.vbits / 8;
  const size_t smem = ((sizeof(Sm) + 15) / 16) * 16 + sizeof(float) * (D * nck * R + (D / 4) * 16 * R) +
                      ((kT * rbk + 15) / 16) * 16 + ((kT * rbv + 15) / 16) * 16;
  cudaError_t e = cudaFuncSetAttribute(decode_main<D, R>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 grid(a.sh.n_splits, static_cast<unsigned>(int64_t(a.sh.batch) * a.sh.hkv * a.sh.row_blocks));
  decode_main<D, R><<<grid, kT, smem, st>>>(a);
  count_launch();
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_main_rows(const DecodeArgs& a, cudaStream_t st) {
  if (D == 64 || D == 128) {
    const char* env = std::getenv("TQ_DECODE_PATH");
    if (!(env && std::strcmp(env, "v1") == 0)) {
      cudaError_t e = cudaSuccess;
      if (try_v2<(D == 64 ? 64 : 128)>(a, st, e)) return e;
    }
  }
  switch (a.sh.rows_per_cta) {
    case 1: return launch_main<D, 1>(a, st);
    case 2: return launch_main<D, 2>(a, st);
    case 4: return launch_main<D, 4>(a, st);
    default: return launch_main<D, 8>(a, st);
  }
}

}  // namespace
}  // namespace tq

extern "C" size_t tq_decode_workspace_bytes(const tq_layout* layout, int32_t batch, int32_t hq, int32_t hkv,
                                            int32_t nq, int64_t n_ctx) {
  if (tq::check_layout(layout) != TQ_OK || batch < 1 || hkv < 1 || hq < hkv || hq % hkv || nq < 1 || n_ctx < 1)
    return 0;
  const tq::DecodeShape sh = tq::make_shape(layout, batch, hq, hkv, nq, n_ctx, n_ctx);
  return std::max(tq::shape_workspace_bytes(sh), tq::tc_decode_workspace_bytes(sh));
}

extern "C" tq_status tq_decode_attention(const tq_layout* layout, const void* q, tq_dtype q_dtype, int32_t batch,
                                         int32_t hq, int32_t hkv, int32_t nq, int64_t n_ctx, int64_t ctx_stride,
                                         const int32_t* q_positions, float rope_base, const tq_planes* k,
                                         const tq_planes* v, const float* PiK, const float* PiV, int64_t pi_stride,
                                         const float* S, const float* cK, const float* cV, float scale, void* out,
                                         tq_dtype out_dtype, float* scores_out, void* workspace,
                                         size_t workspace_bytes, int32_t* d_status, void* stream) {
  using namespace tq;
  clear_error();
  tq_status st = check_layout(layout);
  if (st != TQ_OK) return st;
  const int d = layout->d;
  if (batch < 1 || hkv < 1 || hq < hkv || hq % hkv != 0 || nq < 1)
    return fail(TQ_ERR_INVALID_ARG, "need batch>=1, hkv>=1, hq a multiple of hkv, nq>=1");
  if (n_ctx < 1) return fail(TQ_ERR_INVALID_ARG, "n_ctx must be >= 1 (softmax over an empty cache is undefined)");
  if (ctx_stride != 0 && ctx_stride < n_ctx) return fail(TQ_ERR_INVALID_ARG, "ctx_stride < n_ctx");
  if (!q || !k || !v || !k->idx || !k->sign || !k->norm || !k->rnorm || !v->idx || !v->norm || !PiK || !PiV || !S ||
      !cK || !cV || !out)
    return fail(TQ_ERR_INVALID_ARG, "NULL pointer argument");
  if (q_dtype != TQ_F32 && q_dtype != TQ_BF16) return fail(TQ_ERR_INVALID_ARG, "q_dtype must be TQ_F32 or TQ_BF16");
  if (out_dtype != TQ_F32 && out_dtype != TQ_BF16) return fail(TQ_ERR_INVALID_ARG, "out_dtype must be TQ_F32 or TQ_BF16");
  if (pi_stride < 0) return fail(TQ_ERR_INVALID_ARG, "pi_stride < 0");
  if (!aligned(k->idx, 16) || !aligned(k->sign, 16) || !aligned(v->idx, 16))
    return fail(TQ_ERR_INVALID_ARG, "plane pointers must be 16-byte aligned");
  const DecodeShape sh = make_shape(layout, batch, hq, hkv, nq, n_ctx, ctx_stride);
  const size_t need = std::max(shape_workspace_bytes(sh), tc_decode_workspace_bytes(sh));
  if (!workspace || workspace_bytes < need)
    return fail(TQ_ERR_WORKSPACE, "workspace of %zu bytes needed (got %zu)", need, workspace_bytes);
  if (!aligned(workspace, 256)) return fail(TQ_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  if (sh.n_rows > (int64_t(1) << 31) - 1 || int64_t(batch) * hkv * sh.row_blocks > 65535)
    return fail(TQ_ERR_UNSUPPORTED, "too many query rows / KV streams for one call");
  DecodeArgs a{};
  a.sh = sh;
  a.q = q;
  a.q_dtype = q_dtype == TQ_F32 ? 0 : 1;
  a.q_pos = q_positions;
  a.rope_base = rope_base;
  a.kidx = k->idx;
  a.ksign = k->sign;
  a.knorm = k->norm;
  a.krnorm = k->rnorm;
  a.vidx = v->idx;
  a.vnorm = v->norm;
  a.PiK = PiK;
  a.PiV = PiV;
  a.pi_stride = pi_stride;
  a.S = S;
  a.cK = cK;
  a.cV = cV;
  a.scale = scale;
  a.out = out;
  a.out_dtype = out_dtype == TQ_F32 ? 0 : 1;
  a.scores_out = scores_out;
  a.qs = static_cast<float*>(workspace);
  a.part = reinterpret_cast<float*>(static_cast<char*>(workspace) +
                                    ((size_t(sh.n_rows) * 2 * d * sizeof(float) + 255) / 256) * 256);
  a.d_status = d_status;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  // The fused tensor-core kernel where it applies (TQ_DECODE_PATH=v1|v2
  // selects a CUDA-core kernel instead; all compute the same attention).
  const char* path = std::getenv("TQ_DECODE_PATH");
  const bool cuda_core = path && (std::strcmp(path, "v1") == 0 || std::strcmp(path, "v2") == 0);
  if (!cuda_core && tc_decode_supported(a)) {
    e = tc_decode_launch(a, workspace, s);
  } else {
    e = launch_blk<false>(a, s);
    if (e == cudaSuccess) {
      switch (d) {
        case 64: e = launch_main_rows<64>(a, s); break;
        case 128: e = launch_main_rows<128>(a, s); break;
        case 200: e = launch_main_rows<200>(a, s); break;
        default: return fail(TQ_ERR_UNSUPPORTED, "tq_decode_attention: d=%d not built (64, 128, 200)", d);
      }
    }
    if (e == cudaSuccess) e = launch_blk<true>(a, s);
  }
  if (e != cudaSuccess) return fail(TQ_ERR_CUDA, "tq_decode_attention launch: %s", cudaGetErrorString(e));
  return TQ_OK;
}

// ---------------------------------------------------------------------------
// tq_decode_attention_noalloc: the same attention with the split-KV scratch in
// a fixed device array owned by this library, for callers that cannot
// allocate device memory when they call.
//
// The array lives in this file (64 MiB per device that loads the library, held
// until the process exits). Host code must not hand the array's symbol to a
// kernel: the symbol names a host-side stand-in. The device address is fetched
// with cudaGetSymbolAddress once per device, with that device current, on the
// first call made on it (that first call should therefore happen before any
// stream capture). Every call shares the array and leaves its contents behind;
// the kernels overwrite everything they read, so nothing needs clearing, but
// calls that overlap on the GPU (different streams, or another host thread)
// race on it.
// ---------------------------------------------------------------------------
static constexpr size_t kStaticScratchBytes = size_t(64) << 20;
static __device__ __align__(256) unsigned char g_decode_scratch[kStaticScratchBytes];

namespace tq {
namespace {

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
void* g_scratch_addr[kMaxDevices] = {};

tq_status static_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(TQ_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return fail(TQ_ERR_UNSUPPORTED, "device index %d above %d", dev, kMaxDevices);
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess || !p)
      return fail(TQ_ERR_CUDA, "cudaGetSymbolAddress(decode scratch): %s", cudaGetErrorString(e));
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return TQ_OK;
}

}  // namespace
}  // namespace tq

extern "C" tq_status tq_decode_attention_noalloc(const tq_layout* layout, const void* q, tq_dtype q_dtype,
                                                 int32_t batch, int32_t hq, int32_t hkv, int32_t nq, int64_t n_ctx,
                                                 int64_t ctx_stride, const int32_t* q_positions, float rope_base,
                                                 const tq_planes* k, const tq_planes* v, const float* PiK,
                                                 const float* PiV, int64_t pi_stride, const float* S, const float* cK,
                                                 const float* cV, float scale, void* out, tq_dtype out_dtype,
                                                 float* scores_out, int32_t* d_status, void* stream) {
  using namespace tq;
  clear_error();
  const size_t need = tq_decode_workspace_bytes(layout, batch, hq, hkv, nq, n_ctx);
  if (need == 0) {
    // Let the regular entry point report exactly what is wrong with the arguments.
    return tq_decode_attention(layout, q, q_dtype, batch, hq, hkv, nq, n_ctx, ctx_stride, q_positions, rope_base, k,
                               v, PiK, PiV, pi_stride, S, cK, cV, scale, out, out_dtype, scores_out, nullptr, 0,
                               d_status, stream);
  }
  if (need > kStaticScratchBytes)
    return fail(TQ_ERR_UNSUPPORTED,
                "tq_decode_attention_noalloc: this shape needs %zu bytes of scratch, above the fixed %zu-byte array; "
                "use tq_decode_attention with a caller workspace",
                need, kStaticScratchBytes);
  void* scratch = nullptr;
  tq_status st = static_scratch(&scratch);
  if (st != TQ_OK) return st;
  return tq_decode_attention(layout, q, q_dtype, batch, hq, hkv, nq, n_ctx, ctx_stride, q_positions, rope_base, k, v,
                             PiK, PiV, pi_stride, S, cK, cV, scale, out, out_dtype, scores_out, scratch,
                             kStaticScratchBytes, d_status, stream);
}
