// Decode main kernel, CUDA-core version 2 (included by tq_decode.cu).
//
// One CTA of 128 threads per (KV stream, query-row block, context split),
// tiles of 128 tokens double-buffered in shared memory with cp.async.
//   scores  thread = token. The index row (d*b/8 bytes) is read as words and
//           every code is cut out at a compile-time position; each code costs
//           one 16-byte read of Tk[i][code][0..3] (q_rot_i * c_K[code] for the
//           four query rows) and four adds. Sign bits go four at a time
//           through Ts[nibble][16][0..3].
//   softmax online, per query row, with the running max in shared memory.
//   values  thread = (4 coordinates, token subset). Each token publishes
//           Wt[t][c][r] = p_r(t) ||v_t|| c_V[c]; a coordinate then costs one
//           16-byte read of Wt[t][code] and four adds, in rotated coordinates.
// Rows per CTA R = 4 (or 8); the value codebook is 3-bit.
#pragma once

namespace tq {
namespace {

constexpr int kT2 = 128;   // tokens per tile = threads

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
               "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Bytes [off, off+n) of a packed row held as 32-bit words, n <= 3 or 4 at any
// byte offset (positions are compile-time after unrolling).
template <int OFF>
__device__ __forceinline__ uint32_t bytes_at(const uint32_t* w) {
  constexpr int wi = OFF / 4, sh = 8 * (OFF % 4);
  if constexpr (sh == 0) return w[wi];
  else return __funnelshift_r(w[wi], w[wi + 1], sh);
}

template <int R>
__device__ __forceinline__ void add_rows(float (&acc)[R], const float* e) {
  if constexpr (R % 4 == 0) {
#pragma unroll
    for (int q = 0; q < R / 4; ++q) {
      const float4 x = reinterpret_cast<const float4*>(e)[q];
      acc[4 * q + 0] += x.x;
      acc[4 * q + 1] += x.y;
      acc[4 * q + 2] += x.z;
      acc[4 * q + 3] += x.w;
    }
  } else {
#pragma unroll
    for (int r = 0; r < R; ++r) acc[r] += e[r];
  }
}

template <int D, int R, int KB>
struct V2Smem {
  static constexpr int kRbk = D * KB / 8, kRbv = D * 3 / 8, kSW = D / 32;
  static constexpr int kNck = 1 << KB;
  // Per stage: kidx, vidx, ksign, knorm, krnorm, vnorm (all 16-byte multiples for kT2 = 128).
  static constexpr int kStageBytes = kT2 * (kRbk + kRbv + 4 * kSW + 12);
  static constexpr int kOffTk = 0;                                      // [D][nck][R]
  static constexpr int kOffTs = kOffTk + D * kNck * R * 4;              // [D/4][16][R]
  static constexpr int kOffW = kOffTs + (D / 4) * 16 * R * 4;           // [kT2][8][R]
  static constexpr int kOffStage = kOffW + kT2 * 8 * R * 4;             // 2 stages
  static constexpr int kOffRed = kOffStage + 2 * kStageBytes;           // [4][R] + m, l, corr
  static constexpr int kBytes = kOffRed + (4 * R + 3 * R) * 4;
};

template <int D, int R, int KB>
__global__ void __launch_bounds__(kT2) decode_main_v2(DecodeArgs a) {
  using Sm = V2Smem<D, R, KB>;
  constexpr int kNck = Sm::kNck, kRbk = Sm::kRbk, kRbv = Sm::kRbv, kSW = Sm::kSW;
  extern __shared__ __align__(16) unsigned char sm[];
  float* Tk = reinterpret_cast<float*>(sm + Sm::kOffTk);
  float* Ts = reinterpret_cast<float*>(sm + Sm::kOffTs);
  float* Wt = reinterpret_cast<float*>(sm + Sm::kOffW);
  float* red = reinterpret_cast<float*>(sm + Sm::kOffRed);
  float* s_m = red + 4 * R;
  float* s_l = s_m + R;
  float* s_corr = s_l + R;

  const DecodeShape& sh = a.sh;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int split = blockIdx.x;
  const int64_t unit = blockIdx.y;
  const int rb = static_cast<int>(unit % sh.row_blocks);
  const int64_t bkv = unit / sh.row_blocks;
  const int G = sh.hq / sh.hkv;
  const int kv = static_cast<int>(bkv % sh.hkv);
  const int b = static_cast<int>(bkv / sh.hkv);
  auto qrow = [&](int r) -> int64_t {
    const int rr = rb * R + r;
    return (int64_t(b) * sh.hq + kv * G + rr / sh.nq) * sh.nq + rr % sh.nq;
  };

  // Tables.
  for (int e = tid; e < D * kNck * R; e += kT2) {
    const int r = e % R, c = (e / R) % kNck, i = e / (R * kNck);
    Tk[e] = a.qs[qrow(r) * 2 * D + i] * __ldg(a.cK + c);
  }
  for (int e = tid; e < (D / 4) * 16 * R; e += kT2) {
    const int r = e % R, m = (e / R) % 16, nib = e / (R * 16);
    const float* sv = a.qs + qrow(r) * 2 * D + D + 4 * nib;
    float acc = 0.f;
#pragma unroll
    for (int q = 0; q < 4; ++q) acc += ((m >> q) & 1) ? sv[q] : -sv[q];
    Ts[e] = acc;
  }
  float cV[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) cV[c] = __ldg(a.cV + c);
  if (tid < R) {
    s_m[tid] = -INFINITY;
    s_l[tid] = 0.f;
  }

  const int64_t t_begin = int64_t(split) * sh.chunk;
  const int64_t t_end = (t_begin + sh.chunk < sh.n_ctx) ? t_begin + sh.chunk : sh.n_ctx;
  const int64_t row0 = bkv * sh.ctx_stride;
  const int n_tiles = static_cast<int>((t_end - t_begin + kT2 - 1) / kT2);

  // Stage layout: [kidx | vidx | ksign | knorm | krnorm | vnorm].
  auto stage_ptr = [&](int s) { return sm + Sm::kOffStage + s * Sm::kStageBytes; };
  auto issue = [&](int tile, int s) {
    const int64_t t0 = t_begin + int64_t(tile) * kT2;
    const int nt = static_cast<int>((t_end - t0 < kT2) ? t_end - t0 : kT2);
    unsigned char* st = stage_ptr(s);
    const unsigned char* srcs[6] = {a.kidx + (row0 + t0) * kRbk, a.vidx + (row0 + t0) * kRbv,
                                    reinterpret_cast<const unsigned char*>(a.ksign + (row0 + t0) * kSW),
                                    reinterpret_cast<const unsigned char*>(a.knorm + row0 + t0),
                                    reinterpret_cast<const unsigned char*>(a.krnorm + row0 + t0),
                                    reinterpret_cast<const unsigned char*>(a.vnorm + row0 + t0)};
    const int per[6] = {kRbk, kRbv, 4 * kSW, 4, 4, 4};
    int off = 0;
#pragma unroll
    for (int p = 0; p < 6; ++p) {
      const int bytes = nt * per[p];
      // 16-byte asynchronous copies need a 16-byte aligned source; otherwise
      // (an unusual ctx_stride) the plane is copied byte by byte.
      const int full16 = (reinterpret_cast<uintptr_t>(srcs[p]) & 15) == 0 ? (bytes & ~15) : 0;
      for (int i = tid * 16; i < full16; i += kT2 * 16) cp_async16(st + off + i, srcs[p] + i);
      for (int i = full16 + tid; i < bytes; i += kT2) st[off + i] = srcs[p][i];
      off += kT2 * per[p];
    }
    cp_async_commit();
  };

  // V-phase mapping: lane -> 4 coordinates (4*lane .. 4*lane+3, D/4 quads), warp -> token subset.
  constexpr int kQuads = D / 4;                 // 32 for D=128, 16 for D=64
  constexpr int kSub = kT2 / kQuads;            // token subsets: 4 (D=128) or 8 (D=64)
  const int quad = tid % kQuads, sub = tid / kQuads;
  float acc[4][R];
#pragma unroll
  for (int k = 0; k < 4; ++k)
#pragma unroll
    for (int r = 0; r < R; ++r) acc[k][r] = 0.f;

  const float alpha = static_cast<float>(kSqrtHalfPi / D);
  issue(0, 0);
  for (int tile = 0; tile < n_tiles; ++tile) {
    const int s = tile & 1;
    const int64_t t0 = t_begin + int64_t(tile) * kT2;
    const int nt = static_cast<int>((t_end - t0 < kT2) ? t_end - t0 : kT2);
    __syncthreads();                                   // stage s^1 free, tables ready
    if (tile + 1 < n_tiles) {
      issue(tile + 1, s ^ 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const unsigned char* st = stage_ptr(s);
    const unsigned char* kidx = st;
    const unsigned char* vidx = kidx + kT2 * kRbk;
    const uint32_t* ksign = reinterpret_cast<const uint32_t*>(vidx + kT2 * kRbv);
    const float* knorm = reinterpret_cast<const float*>(ksign + kT2 * kSW);
    const float* krn = knorm + kT2;
    const float* vnorm = krn + kT2;

    // ---- scores (thread = token)
    float score[R];
    if (tid < nt) {
      float ck[R], cs[R];
#pragma unroll
      for (int r = 0; r < R; ++r) ck[r] = cs[r] = 0.f;
      uint32_t w[kRbk / 4 + 1];
      if constexpr (kRbk % 16 == 0) {     // rows start on 16-byte boundaries
#pragma unroll
        for (int q = 0; q < kRbk / 16; ++q) {
          const uint4 x = reinterpret_cast<const uint4*>(kidx + tid * kRbk)[q];
          w[4 * q] = x.x; w[4 * q + 1] = x.y; w[4 * q + 2] = x.z; w[4 * q + 3] = x.w;
        }
      } else {                            // 4-byte aligned rows (d*bits/8 a multiple of 4)
#pragma unroll
        for (int q = 0; q < kRbk / 4; ++q) w[q] = reinterpret_cast<const uint32_t*>(kidx + tid * kRbk)[q];
      }
      w[kRbk / 4] = 0u;
#pragma unroll
      for (int g = 0; g < D / 8; ++g) {
        // Byte offset of group g is KB*g; read it at compile-time position.
        uint32_t word;
        {
          const int off = KB * g;
          const int wi = off >> 2, shf = 8 * (off & 3);
          word = shf == 0 ? w[wi] : __funnelshift_r(w[wi], w[wi + 1], shf);
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int c = (word >> (KB * j)) & (kNck - 1);
          add_rows<R>(ck, Tk + ((8 * g + j) * kNck + c) * R);
        }
      }
      uint32_t sw[kSW];
      if constexpr (kSW % 4 == 0) {
#pragma unroll
        for (int q = 0; q < kSW / 4; ++q) {
          const uint4 y = reinterpret_cast<const uint4*>(ksign + tid * kSW)[q];
          sw[4 * q] = y.x; sw[4 * q + 1] = y.y; sw[4 * q + 2] = y.z; sw[4 * q + 3] = y.w;
        }
      } else {
#pragma unroll
        for (int q = 0; q < kSW; ++q) sw[q] = ksign[tid * kSW + q];
      }
#pragma unroll
      for (int nib = 0; nib < D / 4; ++nib) {
        const int m = (sw[nib >> 3] >> (4 * (nib & 7))) & 15;
        add_rows<R>(cs, Ts + (nib * 16 + m) * R);
      }
      const float kn = knorm[tid], rn = krn[tid];
#pragma unroll
      for (int r = 0; r < R; ++r) score[r] = a.scale * (kn * ck[r] + alpha * rn * cs[r]);
      if (a.scores_out) {
#pragma unroll
        for (int r = 0; r < R; ++r) a.scores_out[qrow(r) * sh.n_ctx + t0 + tid] = score[r];
      }
    } else {
#pragma unroll
      for (int r = 0; r < R; ++r) score[r] = -INFINITY;
    }
    // ---- online softmax over the tile
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const float mx = warp_max(score[r]);
      if (lane == 0) red[warp * R + r] = mx;
    }
    __syncthreads();
    if (tid < R) {
      float mx = red[tid];
#pragma unroll
      for (int w2 = 1; w2 < kT2 / 32; ++w2) mx = fmaxf(mx, red[w2 * R + tid]);
      const float m_old = s_m[tid];
      const float m_new = fmaxf(m_old, mx);
      s_corr[tid] = (m_old == -INFINITY) ? 0.f : __expf(m_old - m_new);
      s_m[tid] = m_new;
    }
    __syncthreads();
    {
      float p[R], psum[R];
      const float vn = (tid < nt) ? vnorm[tid] : 0.f;
#pragma unroll
      for (int r = 0; r < R; ++r) {
        p[r] = (tid < nt) ? __expf(score[r] - s_m[r]) : 0.f;
        psum[r] = warp_sum(p[r]);
        p[r] *= vn;
      }
      // Wt[t][c][r] = p_r ||v|| c_V[c]
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        float* e = Wt + (tid * 8 + c) * R;
        if constexpr (R % 4 == 0) {
#pragma unroll
          for (int q = 0; q < R / 4; ++q)
            reinterpret_cast<float4*>(e)[q] =
                make_float4(p[4 * q] * cV[c], p[4 * q + 1] * cV[c], p[4 * q + 2] * cV[c], p[4 * q + 3] * cV[c]);
        } else {
#pragma unroll
          for (int r = 0; r < R; ++r) e[r] = p[r] * cV[c];
        }
      }
#pragma unroll
      for (int r = 0; r < R; ++r)
        if (lane == 0) red[warp * R + r] = psum[r];
    }
    __syncthreads();
    if (tid < R) {
      float tot = 0.f;
#pragma unroll
      for (int w2 = 0; w2 < kT2 / 32; ++w2) tot += red[w2 * R + tid];
      s_l[tid] = s_l[tid] * s_corr[tid] + tot;
    }
    // ---- values: this thread's 4 coordinates over tokens sub, sub+kSub, ...
    {
      float corr[R];
#pragma unroll
      for (int r = 0; r < R; ++r) corr[r] = s_corr[r];
#pragma unroll
      for (int k = 0; k < 4; ++k)
#pragma unroll
        for (int r = 0; r < R; ++r) acc[k][r] *= corr[r];
      const int bit0 = 12 * quad;                 // 4 codes x 3 bits
      const int wi = bit0 >> 5, shf = bit0 & 31;
      for (int t = sub; t < nt; t += kSub) {
        const uint32_t* vr = reinterpret_cast<const uint32_t*>(vidx + t * kRbv);
        const uint32_t lo = vr[wi];
        const uint32_t hi = (shf + 12 > 32) ? vr[wi + 1] : 0u;
        const uint32_t bits = __funnelshift_r(lo, hi, shf);
        const float* wt = Wt + t * 8 * R;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int c = (bits >> (3 * k)) & 7;
          float tmp[R];
#pragma unroll
          for (int r = 0; r < R; ++r) tmp[r] = 0.f;
          add_rows<R>(tmp, wt + c * R);
#pragma unroll
          for (int r = 0; r < R; ++r) acc[k][r] += tmp[r];
        }
      }
    }
  }
  // ---- partials: reduce the kSub token subsets of each coordinate through shared memory.
  __syncthreads();
  float* part = Wt;     // reuse: [kSub][D][R]
#pragma unroll
  for (int k = 0; k < 4; ++k)
#pragma unroll
    for (int r = 0; r < R; ++r) part[(sub * D + 4 * quad + k) * R + r] = acc[k][r];
  __syncthreads();
  for (int e = tid; e < D * R; e += kT2) {
    const int r = e % R, i = e / R;
    float sum = 0.f;
#pragma unroll
    for (int u = 0; u < kSub; ++u) sum += part[(u * D + i) * R + r];
    a.part[(qrow(r) * sh.n_parts + split) * (D + 2) + i] = sum;
  }
  if (tid < R) {
    float* p = a.part + (qrow(tid) * sh.n_parts + split) * (D + 2);
    p[D] = s_m[tid];
    p[D + 1] = s_l[tid];
  }
}

}  // namespace
}  // namespace tq
