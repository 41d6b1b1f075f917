// tq_search_topk: inner-product search over a corpus stored as 3-bit + QJL
// codes, returning each query's k best database vectors by estimated score.
//
// Sources: sudonull.com "TurboQuant: compresión 6x de LLM KV-cache" (QJL
// keeps inner products; the method serves vector search and RAG) and
// news.hada.io's TurboQuant summary (recall of the true top inner products
// among the approximate top-k, on GloVe d=200). The estimator is the one of
// 7minutos.es "KV cache ... TurboQuant" Etapa 2:
//   est(q, x) = ||x|| <Pi q, c[idx_x]> + sqrt(pi/2)/d ||r_x|| <S Pi q, 2 sign_x - 1>.
// Ranking: decreasing score; equal scores by increasing database index.
//
// Launches: (1) q_rot = Pi q and s = S q_rot per query; (2) per (query block
// of 8, corpus chunk) a CTA scores every vector against its queries through
// shared-memory tables (code LUT per coordinate, sign LUT per nibble) and
// keeps each query's best k in a warp-wide sorted list (lane j = j-th best);
// (3) one warp per query merges the chunk lists.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>

#include "tq_device.cuh"
#include "tq_internal.h"

namespace tq {
namespace {

using namespace dev;

constexpr int kSThreads = 256;
constexpr int kSRows = 8;          // queries per CTA
constexpr int kChunk = 8192;       // corpus vectors per CTA
constexpr int kMaxK = 32;
constexpr int kServeBlock = 16384;  // queries per pass with the workspace tq_search_workspace_bytes reports

struct SearchArgs {
  int d, bits, nq, k;
  int64_t n_db;
  int n_chunks;
  const void* q;
  int q_dtype;
  const uint8_t* idx;
  const uint32_t* sign;
  const float* norm;
  const float* rnorm;
  const float* Pi;
  const float* S;
  const float* cent;
  float* qs;          // [nq][2][d]
  float* cand_s;      // [nq][n_chunks][k]
  int64_t* cand_i;    // [nq][n_chunks][k]
  int64_t* top_idx;
  float* top_s;
};

__global__ void search_prologue(SearchArgs a) {
  extern __shared__ double sp_smem[];
  const int d = a.d;
  double* qd = sp_smem;
  float* qr = reinterpret_cast<float*>(sp_smem + d);
  const int64_t row = blockIdx.x;
  for (int i = threadIdx.x; i < d; i += blockDim.x) qd[i] = load_elem(a.q, a.q_dtype, row * d + i);
  __syncthreads();
  for (int i = threadIdx.x; i < d; i += blockDim.x) {
    double acc = 0.0;
    for (int j = 0; j < d; ++j) acc = fma(static_cast<double>(__ldg(a.Pi + int64_t(i) * d + j)), qd[j], acc);
    qr[i] = static_cast<float>(acc);
    a.qs[row * 2 * d + i] = static_cast<float>(acc);
  }
  __syncthreads();
  for (int i = threadIdx.x; i < d; i += blockDim.x) {
    double acc = 0.0;
    for (int j = 0; j < d; ++j) acc = fma(static_cast<double>(__ldg(a.S + int64_t(i) * d + j)), double(qr[j]), acc);
    a.qs[row * 2 * d + d + i] = static_cast<float>(acc);
  }
}

// (score, index) ordering: higher score first, lower index on ties.
__device__ __forceinline__ bool better(float s1, int64_t i1, float s2, int64_t i2) {
  return s1 > s2 || (s1 == s2 && i1 < i2);
}

// Warp-wide sorted list of the k best (lane j holds the j-th best; lanes >= k
// and empty slots hold -inf). Inserts (s, i) if it beats the k-th entry.
__device__ __forceinline__ void list_insert(float& ls, int64_t& li, int k, float s, int64_t i) {
  const int lane = threadIdx.x & 31;
  const float ks = __shfl_sync(0xffffffffu, ls, k - 1);
  const int64_t ki = __shfl_sync(0xffffffffu, li, k - 1);
  if (!better(s, i, ks, ki)) return;
  const bool after = better(s, i, ls, li);                 // new entry sits at or before this lane
  const unsigned m = __ballot_sync(0xffffffffu, after);
  const int pos = m ? __ffs(m) - 1 : 32;
  const float ps = __shfl_up_sync(0xffffffffu, ls, 1);
  const int64_t pi = __shfl_up_sync(0xffffffffu, li, 1);
  if (lane > pos) {
    ls = ps;
    li = pi;
  } else if (lane == pos) {
    ls = s;
    li = i;
  }
}

template <int D>
__global__ void __launch_bounds__(kSThreads) search_main(SearchArgs a) {
  extern __shared__ __align__(16) unsigned char sm_raw[];
  const int nc = 1 << a.bits;
  const int rb = D * a.bits / 8;
  constexpr int kSW = (D + 31) / 32;
  float* Tk = reinterpret_cast<float*>(sm_raw);                     // [D][nc][8]
  float* Ts = Tk + D * nc * kSRows;                                 // [D/4][16][8]
  float* wl_s = Ts + (D / 4) * 16 * kSRows;                         // [8 warps][8 rows][32]
  int64_t* wl_i = reinterpret_cast<int64_t*>(wl_s + 8 * kSRows * 32);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int chunk = blockIdx.x;
  const int q0 = blockIdx.y * kSRows;
  const int nr = min(kSRows, a.nq - q0);
  for (int e = tid; e < D * nc * kSRows; e += kSThreads) {
    const int r = e % kSRows, c = (e / kSRows) % nc, i = e / (kSRows * nc);
    Tk[e] = r < nr ? a.qs[int64_t(q0 + r) * 2 * D + i] * __ldg(a.cent + c) : 0.f;
  }
  for (int e = tid; e < (D / 4) * 16 * kSRows; e += kSThreads) {
    const int r = e % kSRows, m = (e / kSRows) % 16, nib = e / (kSRows * 16);
    float acc = 0.f;
    if (r < nr) {
      const float* sv = a.qs + int64_t(q0 + r) * 2 * D + D + 4 * nib;
#pragma unroll
      for (int q = 0; q < 4; ++q) acc += ((m >> q) & 1) ? sv[q] : -sv[q];
    }
    Ts[e] = acc;
  }
  __syncthreads();
  // Each warp keeps, for each of the 8 queries, its own sorted top-k.
  float ls[kSRows];
  int64_t li[kSRows];
#pragma unroll
  for (int r = 0; r < kSRows; ++r) {
    ls[r] = -INFINITY;
    li[r] = INT64_MAX;
  }
  const float alpha = static_cast<float>(kSqrtHalfPi / D);
  const int64_t v_begin = int64_t(chunk) * kChunk;
  const int64_t v_end = min(a.n_db, v_begin + kChunk);
  for (int64_t v0 = v_begin; v0 < v_end; v0 += kSThreads) {
    const int64_t v = v0 + tid;
    float score[kSRows];
    if (v < v_end) {
      float ck[kSRows], cs[kSRows];
#pragma unroll
      for (int r = 0; r < kSRows; ++r) ck[r] = cs[r] = 0.f;
      const uint8_t* row = a.idx + v * rb;
      for (int g = 0; g < D / 8; ++g) {
        uint32_t word = 0;
        for (int b = 0; b < a.bits; ++b) word |= static_cast<uint32_t>(__ldg(row + g * a.bits + b)) << (8 * b);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int c = (word >> (a.bits * j)) & (nc - 1);
          const float4* e = reinterpret_cast<const float4*>(Tk + ((8 * g + j) * nc + c) * kSRows);
          const float4 e0 = e[0], e1 = e[1];
          ck[0] += e0.x; ck[1] += e0.y; ck[2] += e0.z; ck[3] += e0.w;
          ck[4] += e1.x; ck[5] += e1.y; ck[6] += e1.z; ck[7] += e1.w;
        }
      }
      const uint32_t* srow = a.sign + v * kSW;
      for (int w = 0; w < kSW; ++w) {
        const uint32_t sw = __ldg(srow + w);
        const int nib_end = min(8, D / 4 - w * 8);
        for (int t = 0; t < nib_end; ++t) {
          const int m = (sw >> (4 * t)) & 15;
          const float4* e = reinterpret_cast<const float4*>(Ts + ((w * 8 + t) * 16 + m) * kSRows);
          const float4 e0 = e[0], e1 = e[1];
          cs[0] += e0.x; cs[1] += e0.y; cs[2] += e0.z; cs[3] += e0.w;
          cs[4] += e1.x; cs[5] += e1.y; cs[6] += e1.z; cs[7] += e1.w;
        }
      }
      const float kn = __ldg(a.norm + v), rn = __ldg(a.rnorm + v);
#pragma unroll
      for (int r = 0; r < kSRows; ++r) score[r] = kn * ck[r] + alpha * rn * cs[r];
    } else {
#pragma unroll
      for (int r = 0; r < kSRows; ++r) score[r] = -INFINITY;
    }
    // Insert this warp's 32 candidates per query (only those above the k-th).
#pragma unroll
    for (int r = 0; r < kSRows; ++r) {
      const float kth = __shfl_sync(0xffffffffu, ls[r], a.k - 1);
      const int64_t kti = __shfl_sync(0xffffffffu, li[r], a.k - 1);
      unsigned m = __ballot_sync(0xffffffffu, v < v_end && better(score[r], v, kth, kti));
      while (m) {
        const int src = __ffs(m) - 1;
        m &= m - 1;
        const float s = __shfl_sync(0xffffffffu, score[r], src);
        const int64_t i = __shfl_sync(0xffffffffu, v, src);
        list_insert(ls[r], li[r], a.k, s, i);
      }
    }
  }
  // Merge the 8 warps' lists per query; warp r handles query r.
#pragma unroll
  for (int r = 0; r < kSRows; ++r) {
    wl_s[(warp * kSRows + r) * 32 + lane] = ls[r];
    wl_i[(warp * kSRows + r) * 32 + lane] = li[r];
  }
  __syncthreads();
  if (warp < nr) {
    const int r = warp;
    float ms = -INFINITY;
    int64_t mi = INT64_MAX;
    for (int w = 0; w < kSThreads / 32; ++w) {
      for (int j = 0; j < a.k; ++j) {
        const float s = wl_s[(w * kSRows + r) * 32 + j];
        const int64_t i = wl_i[(w * kSRows + r) * 32 + j];
        if (s > -INFINITY) list_insert(ms, mi, a.k, s, i);
      }
    }
    if (lane < a.k) {
      const int64_t o = (int64_t(q0 + r) * a.n_chunks + chunk) * a.k + lane;
      a.cand_s[o] = ms;
      a.cand_i[o] = mi;
    }
  }
}

__global__ void search_merge(SearchArgs a) {
  const int lane = threadIdx.x & 31;
  const int64_t q = int64_t(blockIdx.x) * (blockDim.x / 32) + (threadIdx.x >> 5);
  if (q >= a.nq) return;
  float ms = -INFINITY;
  int64_t mi = INT64_MAX;
  const int64_t n = int64_t(a.n_chunks) * a.k;
  for (int64_t base = 0; base < n; base += 32) {
    const int64_t j = base + lane;
    const float s = j < n ? a.cand_s[q * n + j] : -INFINITY;
    const int64_t i = j < n ? a.cand_i[q * n + j] : INT64_MAX;
    const float kth = __shfl_sync(0xffffffffu, ms, a.k - 1);
    const int64_t kti = __shfl_sync(0xffffffffu, mi, a.k - 1);
    unsigned m = __ballot_sync(0xffffffffu, s > -INFINITY && better(s, i, kth, kti));
    while (m) {
      const int src = __ffs(m) - 1;
      m &= m - 1;
      list_insert(ms, mi, a.k, __shfl_sync(0xffffffffu, s, src), __shfl_sync(0xffffffffu, i, src));
    }
  }
  if (lane < a.k) {
    a.top_idx[q * a.k + lane] = mi == INT64_MAX ? -1 : mi;
    a.top_s[q * a.k + lane] = ms;
  }
}

// Merge of two per-query top-k lists (one warp per query): list A enters as
// is, B's entries are inserted; ids are shifted by each list's offset, and -1
// (an empty slot) never enters. Inputs are read before any output is written,
// so the output may alias either input.
__global__ void search_merge_lists(int nq, int k, const int64_t* ia, const float* sa, int64_t oa, const int64_t* ib,
                                   const float* sb, int64_t ob, int64_t* io, float* so) {
  const int lane = threadIdx.x & 31;
  const int64_t q = int64_t(blockIdx.x) * (blockDim.x / 32) + (threadIdx.x >> 5);
  if (q >= nq) return;
  const int64_t base = q * k;
  const int64_t a_i = lane < k ? ia[base + lane] : -1;
  const float a_s = lane < k ? sa[base + lane] : -INFINITY;
  const int64_t b_i = lane < k ? ib[base + lane] : -1;
  const float b_s = lane < k ? sb[base + lane] : -INFINITY;
  float ms = a_i >= 0 ? a_s : -INFINITY;
  int64_t mi = a_i >= 0 ? a_i + oa : INT64_MAX;
  const int64_t gb = b_i >= 0 ? b_i + ob : INT64_MAX;
  unsigned m = __ballot_sync(0xffffffffu, b_i >= 0);
  while (m) {
    const int src = __ffs(m) - 1;
    m &= m - 1;
    list_insert(ms, mi, k, __shfl_sync(0xffffffffu, b_s, src), __shfl_sync(0xffffffffu, gb, src));
  }
  if (lane < k) {
    io[base + lane] = mi == INT64_MAX ? -1 : mi;
    so[base + lane] = ms;
  }
}

size_t search_ws(int d, int nq, int64_t n_db, int k) {
  const int64_t chunks = (n_db + kChunk - 1) / kChunk;
  const size_t qs = ((size_t(nq) * 2 * d * 4 + 255) / 256) * 256;
  const size_t cs = ((size_t(nq) * chunks * k * 4 + 255) / 256) * 256;
  const size_t ci = size_t(nq) * chunks * k * 8;
  return qs + cs + ci;
}

}  // namespace
}  // namespace tq

extern "C" size_t tq_search_workspace_bytes(const tq_layout* layout, int32_t n_queries, int64_t n_db, int32_t k) {
  if (tq::check_layout(layout) != TQ_OK || n_queries < 1 || n_db < 1 || k < 1 || k > tq::kMaxK) return 0;
  return tq::search_ws(layout->d, n_queries < tq::kServeBlock ? n_queries : tq::kServeBlock, n_db, k);
}

extern "C" tq_status tq_search_topk(const tq_layout* layout, const void* q, tq_dtype q_dtype, int32_t n_queries,
                                    const tq_planes* db, int64_t n_db, const float* Pi, const float* S,
                                    const float* centroids, int32_t k, int64_t* top_idx, float* top_scores,
                                    void* workspace, size_t workspace_bytes, void* stream) {
  using namespace tq;
  clear_error();
  tq_status st = check_layout(layout);
  if (st != TQ_OK) return st;
  const int d = layout->d;
  if (n_queries < 1 || n_db < 1) return fail(TQ_ERR_INVALID_ARG, "need n_queries >= 1 and n_db >= 1");
  if (k < 1 || k > kMaxK || k > n_db) return fail(TQ_ERR_INVALID_ARG, "k must be in [1, min(32, n_db)] (got %d)", k);
  if (!q || !db || !db->idx || !db->sign || !db->norm || !db->rnorm || !Pi || !S || !centroids || !top_idx ||
      !top_scores)
    return fail(TQ_ERR_INVALID_ARG, "NULL pointer argument");
  if (q_dtype != TQ_F32 && q_dtype != TQ_BF16) return fail(TQ_ERR_INVALID_ARG, "q_dtype must be TQ_F32 or TQ_BF16");
  // Queries run in blocks of as many as the workspace holds (one pass when it
  // holds them all).
  if (!workspace || workspace_bytes < search_ws(d, 1, n_db, k))
    return fail(TQ_ERR_WORKSPACE, "workspace of at least %zu bytes needed (got %zu)", search_ws(d, 1, n_db, k),
                workspace_bytes);
  if (!aligned(workspace, 256)) return fail(TQ_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  int qb = n_queries < kServeBlock ? n_queries : kServeBlock;
  while (qb > 1 && search_ws(d, qb, n_db, k) > workspace_bytes) qb = (qb + 1) / 2;
  while (qb < n_queries && search_ws(d, qb + 1, n_db, k) <= workspace_bytes && qb < kServeBlock) ++qb;
  const int n_chunks = static_cast<int>((n_db + kChunk - 1) / kChunk);
  if (d != 64 && d != 128 && d != 200) return fail(TQ_ERR_UNSUPPORTED, "tq_search_topk: d=%d not built (64, 128, 200)", d);
  const size_t elem = q_dtype == TQ_F32 ? 4 : 2;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaSuccess;
  for (int q0 = 0; q0 < n_queries && e == cudaSuccess; q0 += qb) {
    const int nb = n_queries - q0 < qb ? n_queries - q0 : qb;
    SearchArgs a{};
    a.d = d;
    a.bits = layout->key_bits;
    a.nq = nb;
    a.k = k;
    a.n_db = n_db;
    a.n_chunks = n_chunks;
    a.q = static_cast<const char*>(q) + size_t(q0) * d * elem;
    a.q_dtype = q_dtype == TQ_F32 ? 0 : 1;
    a.idx = db->idx;
    a.sign = db->sign;
    a.norm = db->norm;
    a.rnorm = db->rnorm;
    a.Pi = Pi;
    a.S = S;
    a.cent = centroids;
    char* w = static_cast<char*>(workspace);
    a.qs = reinterpret_cast<float*>(w);
    w += ((size_t(nb) * 2 * d * 4 + 255) / 256) * 256;
    a.cand_s = reinterpret_cast<float*>(w);
    w += ((size_t(nb) * n_chunks * k * 4 + 255) / 256) * 256;
    a.cand_i = reinterpret_cast<int64_t*>(w);
    a.top_idx = top_idx + int64_t(q0) * k;
    a.top_s = top_scores + int64_t(q0) * k;
    search_prologue<<<nb, 128, d * sizeof(double) + d * sizeof(float), s>>>(a);
    count_launch();
    e = cudaGetLastError();
    if (e == cudaSuccess) {
      const int nc = 1 << a.bits;
      const size_t smem = sizeof(float) * (d * nc * kSRows + (d / 4) * 16 * kSRows + 8 * kSRows * 32) +
                          sizeof(int64_t) * 8 * kSRows * 32;
      dim3 grid(n_chunks, (nb + kSRows - 1) / kSRows);
      switch (d) {
        case 64:
          cudaFuncSetAttribute(search_main<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
          search_main<64><<<grid, kSThreads, smem, s>>>(a);
          break;
        case 128:
          cudaFuncSetAttribute(search_main<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
          search_main<128><<<grid, kSThreads, smem, s>>>(a);
          break;
        default:
          cudaFuncSetAttribute(search_main<200>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
          search_main<200><<<grid, kSThreads, smem, s>>>(a);
          break;
      }
      count_launch();
      e = cudaGetLastError();
    }
    if (e == cudaSuccess) {
      search_merge<<<(nb + 3) / 4, 128, 0, s>>>(a);
      count_launch();
      e = cudaGetLastError();
    }
  }
  if (e != cudaSuccess) return fail(TQ_ERR_CUDA, "tq_search_topk launch: %s", cudaGetErrorString(e));
  return TQ_OK;
}

extern "C" tq_status tq_search_merge_topk(int32_t n_queries, int32_t k, const int64_t* idx_a, const float* scores_a,
                                         int64_t offset_a, const int64_t* idx_b, const float* scores_b,
                                         int64_t offset_b, int64_t* idx_out, float* scores_out, void* stream) {
  using namespace tq;
  clear_error();
  if (n_queries < 0) return fail(TQ_ERR_INVALID_ARG, "n_queries < 0");
  if (n_queries == 0) return TQ_OK;
  if (k < 1 || k > kMaxK) return fail(TQ_ERR_INVALID_ARG, "k must be in [1, 32] (got %d)", k);
  if (!idx_a || !scores_a || !idx_b || !scores_b || !idx_out || !scores_out)
    return fail(TQ_ERR_INVALID_ARG, "NULL pointer argument");
  if (offset_a < 0 || offset_b < 0) return fail(TQ_ERR_INVALID_ARG, "offsets must be >= 0");
  search_merge_lists<<<(n_queries + 3) / 4, 128, 0, static_cast<cudaStream_t>(stream)>>>(
      n_queries, k, idx_a, scores_a, offset_a, idx_b, scores_b, offset_b, idx_out, scores_out);
  count_launch();
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(TQ_ERR_CUDA, "tq_search_merge_topk launch: %s", cudaGetErrorString(e));
  return TQ_OK;
}
