// Row statistics of temperature softmax (the bandwidth-bound hot loop) and
// the finalisation used by spec_softmax_T.
//
// Temperature softmax of target and draft logit rows, z = x / T: the
// verifier samples both with one sampling filter ("DBLAST: Dependent Block
// Drafting for Stochastic Speculative Decoding", Pith review, "Assumptions";
// target sampling at T = 1.5 in "What would settle it").
//
// Design. A persistent grid of G blocks (a multiple of the SM count) splits
// the flattened units of every row evenly, so every block streams the same
// number of bytes whatever the row count; a block's range covers a tail of
// one row, whole rows, and a head of another. Each thread keeps an online
// (max, sum of 2^((x - max) log2e / T)) over its 16-byte vectors: a group of
// U vectors is loaded at once, its maximum taken exactly on the raw bf16
// pairs, then one exponential per element. Blocks write one partial per
// (row, block); consumers merge the few partials of a row.
#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace specv {

constexpr int kUnroll = 4;  // 16-byte vectors in flight per thread per group

// Geometry of the verify walk, built in shared memory by every block:
// rowoff[b] first walk row of request b (rowoff[B] = total), base[b] target
// row of its position 0. Request b owns (K+1)*l walk rows: l target rows,
// then K draft categories of l rows each, l = verified length.
struct Walk {
  const int* rowoff;
  const int* base;
};

// Row r of the walk and the address of the drafted token of its position
// (nullptr outside verify mode). The token itself is loaded by the caller,
// which uses it only after the row's first data has arrived.
template <int DT>
__device__ __forceinline__ const char* locate(const RowSpace& rs, const Walk& w, int64_t r, const int32_t*& tokp) {
  constexpr int64_t esz = Elem<DT>::kBytes;
  tokp = nullptr;
  if (!rs.verify) return static_cast<const char*>(rs.target) + r * rs.stride * esz;
  int lo = 0, hi = rs.B - 1;  // last request whose first row is <= r
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (w.rowoff[mid] <= r) lo = mid; else hi = mid - 1;
  }
  const int b = lo;
  const int q = static_cast<int>(r - w.rowoff[b]);
  const int l = (w.rowoff[b + 1] - w.rowoff[b]) / (rs.K + 1);
  if (q < l) {
    tokp = rs.tokens + static_cast<int64_t>(b) * rs.L + q;
    return static_cast<const char*>(rs.target) + (static_cast<int64_t>(w.base[b]) + q) * rs.stride * esz;
  }
  const int q2 = q - l, z = q2 / l, i = q2 - z * l;
  tokp = rs.tokens + static_cast<int64_t>(b) * rs.L + i;
  return static_cast<const char*>(rs.draft) + ((static_cast<int64_t>(b) * rs.K + z) * rs.L + i) * rs.stride * esz;
}

__device__ __forceinline__ int load_token(const int32_t* tokp) { return tokp ? __ldg(tokp) : -1; }

// Element `idx` (0..E-1) of a 16-byte vector.
template <int DT>
__device__ __forceinline__ float vec_elem(const uint4& h, int idx) {
  if constexpr (DT == 1) {
    const int wi = idx >> 1;
    const uint32_t wd = wi == 0 ? h.x : wi == 1 ? h.y : wi == 2 ? h.z : h.w;
    return (idx & 1) ? bf16hi(wd) : bf16lo(wd);
  } else {
    return __uint_as_float(idx == 0 ? h.x : idx == 1 ? h.y : idx == 2 ? h.z : h.w);
  }
}

// If this thread's group (units u, u + kThreads, ...) holds the drafted token,
// take its logit from the registers.
template <int DT, int N>
__device__ __forceinline__ void pick_token(const uint4 (&v)[N], int u, int tok, float& xv, bool& hit) {
  constexpr int E = Elem<DT>::kPerVec;
  if (tok < 0) return;
  const int rel = tok / E - u;
  if (rel >= 0 && rel < N * kThreads && rel % kThreads == 0) {
    uint4 h = v[0];
#pragma unroll
    for (int t = 1; t < N; ++t)
      if (rel == t * kThreads) h = v[t];
    xv = vec_elem<DT>(h, tok - (tok / E) * E);
    hit = true;
  }
}

// Vector path: each segment (the block's part of one row) streams groups of
// kUnroll 16-byte vectors per thread, then single vectors, and ends with one
// block merge. The drafted token is loaded with the row's first data and
// used only after it, so the stream never waits on it.
template <int DT>
__device__ __forceinline__ void walk_vec(const RowSpace& rs, const Walk& w, int64_t Vu, int64_t e0, int64_t e1,
                                         float k, float2* __restrict__ part, float2* red) {
  const int tid = threadIdx.x;
  for (int64_t e = e0; e < e1;) {
    const int64_t r = e / Vu;
    const int u0 = static_cast<int>(e - r * Vu), u1 = static_cast<int>(min(e1, (r + 1) * Vu) - r * Vu);
    const int32_t* tokp;
    const uint4* rv = reinterpret_cast<const uint4*>(locate<DT>(rs, w, r, tokp));
    const int tok = load_token(tokp);  // out of range: matches no unit of the row
    float m = -INFINITY, s = 0.f, xv = 0.f;
    bool hit = false;
    int u = u0 + tid;
    for (; u + (kUnroll - 1) * kThreads < u1; u += kUnroll * kThreads) {
      uint4 v[kUnroll];
#pragma unroll
      for (int t = 0; t < kUnroll; ++t) v[t] = ldg16(rv + u + t * kThreads);
      fold_vectors<DT, kUnroll>(v, m, s, k);
      pick_token<DT, kUnroll>(v, u, tok, xv, hit);
    }
    for (; u < u1; u += kThreads) {
      const uint4 v[1] = {ldg16(rv + u)};
      fold_vectors<DT, 1>(v, m, s, k);
      pick_token<DT, 1>(v, u, tok, xv, hit);
    }
    if (hit) rs.xg[r] = xv;
    block_merge(m, s, k, red);
    if (tid == 0) part[blockIdx.x + r] = make_float2(m, s);
    e = r * Vu + u1;
  }
}

// Scalar path (rows that are not 16-byte vectors): one segment at a time.
template <int DT>
__device__ __forceinline__ void walk_scalar(const RowSpace& rs, const Walk& w, int64_t Vu, int64_t e0, int64_t e1,
                                            float k, float2* __restrict__ part, float2* red) {
  for (int64_t e = e0; e < e1;) {
    const int64_t r = e / Vu;
    const int64_t se = min(e1, (r + 1) * Vu);
    const int32_t* tokp;
    const char* row = locate<DT>(rs, w, r, tokp);
    const int tok = load_token(tokp);
    float m = -INFINITY, s = 0.f;
    for (int64_t u = e - r * Vu + threadIdx.x; u < se - r * Vu; u += kThreads) {
      const float x = Elem<DT>::at(row, u);
      if (x > m) {
        s *= ex2((m - x) * k);
        m = x;
      }
      if (m != -INFINITY) s += ex2((x - m) * k);
      if (u == tok) rs.xg[r] = x;
    }
    block_merge(m, s, k, red);
    if (threadIdx.x == 0) part[blockIdx.x + r] = make_float2(m, s);
    e = se;
  }
}

template <int DT, bool VEC>
__global__ void __launch_bounds__(kThreads) k_row_stats(RowSpace rs, int64_t Vu, int G, float k,
                                                        float2* __restrict__ part) {
  extern __shared__ int walk_smem[];  // verify mode: rowoff[B + 1], base[B]
  __shared__ float2 red[kWarps];
  __shared__ int tmp[kWarps + 1];
  pdl_wait();
  pdl_trigger();
  int64_t nrows;
  Walk w{walk_smem, walk_smem + rs.B + 1};
  if (rs.verify) {
    int* rowoff = walk_smem;
    int* base = walk_smem + rs.B + 1;
    for (int b = threadIdx.x; b < rs.B; b += kThreads) {
      int l = rs.vlen ? rs.vlen[b] : rs.L;
      if (l < 0 || l > rs.L) l = 0;  // flagged by the sampling kernel
      rowoff[b] = (rs.K + 1) * l;
      base[b] = rs.row_off ? rs.row_off[b] : b * (rs.L + 1);
    }
    __syncthreads();
    nrows = block_exclusive_scan(rowoff, rs.B, tmp);
    if (threadIdx.x == 0) rowoff[rs.B] = static_cast<int>(nrows);
    __syncthreads();
  } else {
    nrows = rs.rows;
  }
  const int64_t N = nrows * Vu;
  const int64_t e0 = split_start(blockIdx.x, N, G), e1 = split_start(blockIdx.x + 1, N, G);
  if (e0 >= e1) return;  // empty share (N < grid): no partials
  if constexpr (VEC) walk_vec<DT>(rs, w, Vu, e0, e1, k, part, red);
  else walk_scalar<DT>(rs, w, Vu, e0, e1, k, part, red);
}

// Merge the partials of row r.
__device__ __forceinline__ void merge_row(const float2* part, int64_t r, int64_t Vu, int64_t N, int G, float k,
                                          float& m, float& s) {
  const int64_t c0 = split_owner(r * Vu, N, G), c1 = split_owner((r + 1) * Vu - 1, N, G);
  m = -INFINITY;
  s = 0.f;
  for (int64_t c = c0; c <= c1; ++c) {
    if (split_start(c + 1, N, G) == split_start(c, N, G)) continue;  // empty share (N < grid): no partial
    const float2 p = part[c + r];
    ms_merge(m, s, p.x, p.y, k);
  }
}

__global__ void __launch_bounds__(kThreads) k_softmax_stats(int64_t rows, int64_t Vu, int G, float k, float T,
                                                            const float2* __restrict__ part, float* row_max,
                                                            float* row_lse) {
  pdl_wait();
  pdl_trigger();
  const int64_t r = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x;
  if (r >= rows) return;
  float m, s;
  merge_row(part, r, Vu, rows * Vu, G, k, m, s);
  row_max[r] = m / T;
  row_lse[r] = m / T + logf(s);
}

template <int DT, bool VEC>
__global__ void __launch_bounds__(kThreads) k_softmax_probs(const void* logits, int64_t rows, int64_t V,
                                                            int64_t stride, int64_t Vu, int G, float k, float T,
                                                            const float2* __restrict__ part, float* row_max,
                                                            float* row_lse, float* probs) {
  __shared__ float sm_m, sm_inv;
  pdl_wait();
  pdl_trigger();
  const int64_t chunks = (Vu + static_cast<int64_t>(kThreads) * 4 - 1) / (static_cast<int64_t>(kThreads) * 4);
  const int64_t r = blockIdx.x / chunks, chunk = blockIdx.x % chunks;
  if (threadIdx.x == 0) {
    float m, s;
    merge_row(part, r, Vu, rows * Vu, G, k, m, s);
    sm_m = m;
    sm_inv = 1.f / s;
    if (chunk == 0) {
      row_max[r] = m / T;
      row_lse[r] = m / T + logf(s);
    }
  }
  __syncthreads();
  const float m = sm_m, inv = sm_inv;
  const char* row = static_cast<const char*>(logits) + r * stride * Elem<DT>::kBytes;
  float* out = probs + r * V;
  for (int64_t u = chunk * kThreads + threadIdx.x; u < Vu; u += chunks * kThreads) {
    if constexpr (VEC) {
      constexpr int E = Elem<DT>::kPerVec;
      float x[E];
      Elem<DT>::unpack(ldg16(reinterpret_cast<const uint4*>(row) + u), x);
      float4* o = reinterpret_cast<float4*>(out + u * E);
#pragma unroll
      for (int h = 0; h < E / 4; ++h)
        o[h] = make_float4(ex2((x[4 * h] - m) * k) * inv, ex2((x[4 * h + 1] - m) * k) * inv,
                           ex2((x[4 * h + 2] - m) * k) * inv, ex2((x[4 * h + 3] - m) * k) * inv);
    } else {
      out[u] = ex2((Elem<DT>::at(row, u) - m) * k) * inv;
    }
  }
}

// ------------------------------------------------------------------- host side

static float log2e_over(float T) { return static_cast<float>(1.4426950408889634 / static_cast<double>(T)); }

template <int DT, bool VEC>
static int occupancy_of() {
  int dev = 0, occ = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 1;
  static std::mutex mu;
  static int cache[64] = {0};
  std::lock_guard<std::mutex> lock(mu);
  if (dev < 64 && cache[dev]) return cache[dev];
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k_row_stats<DT, VEC>, kThreads, 16384) != cudaSuccess ||
      occ < 1)
    occ = 1;
  int sms = 0;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int per_sm = std::max(1, std::min(occ, kGMax / std::max(1, sms)));
  const int g = std::max(1, sms * per_sm);
  if (dev < 64) cache[dev] = g;
  return g;
}

int stats_grid(int dtype, bool vec, int64_t max_units) {
  int g;
  if (dtype == 0) g = vec ? occupancy_of<0, true>() : occupancy_of<0, false>();
  else g = vec ? occupancy_of<1, true>() : occupancy_of<1, false>();
  const int64_t need = (max_units + kThreads - 1) / kThreads;  // at least one unit per thread
  return static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(g, need)));
}

cudaError_t launch_row_stats(const RowSpace& rs, int dtype, bool vec, int64_t V, float T, int G, float2* part,
                             cudaStream_t st) {
  const int64_t Vu = units_per_row(V, dtype, vec);
  const float k = log2e_over(T);
  const size_t smem = rs.verify ? static_cast<size_t>(2 * rs.B + 1) * sizeof(int) : 0;
  const dim3 grid(G), block(kThreads);
  if (dtype == 0)
    return vec ? launch_pdl(k_row_stats<0, true>, grid, block, smem, st, rs, Vu, G, k, part)
               : launch_pdl(k_row_stats<0, false>, grid, block, smem, st, rs, Vu, G, k, part);
  return vec ? launch_pdl(k_row_stats<1, true>, grid, block, smem, st, rs, Vu, G, k, part)
             : launch_pdl(k_row_stats<1, false>, grid, block, smem, st, rs, Vu, G, k, part);
}

cudaError_t launch_softmax_finalize(const void* logits, int dtype, bool vec, int64_t rows, int64_t V,
                                    int64_t stride, float T, int G, const float2* part, float* row_max,
                                    float* row_lse, float* probs, cudaStream_t st) {
  const int64_t Vu = units_per_row(V, dtype, vec);
  const float k = log2e_over(T);
  if (!probs) {
    const dim3 grid(static_cast<unsigned>((rows + kThreads - 1) / kThreads));
    return launch_pdl(k_softmax_stats, grid, dim3(kThreads), 0, st, rows, Vu, G, k, T, part, row_max, row_lse);
  }
  const int64_t per_block = static_cast<int64_t>(kThreads) * 4;
  const dim3 grid(static_cast<unsigned>(rows * ((Vu + per_block - 1) / per_block)));
  const dim3 block(kThreads);
  if (dtype == 0)
    return vec ? launch_pdl(k_softmax_probs<0, true>, grid, block, 0, st, logits, rows, V, stride, Vu, G, k, T,
                            part, row_max, row_lse, probs)
               : launch_pdl(k_softmax_probs<0, false>, grid, block, 0, st, logits, rows, V, stride, Vu, G, k, T,
                            part, row_max, row_lse, probs);
  return vec ? launch_pdl(k_softmax_probs<1, true>, grid, block, 0, st, logits, rows, V, stride, Vu, G, k, T,
                          part, row_max, row_lse, probs)
             : launch_pdl(k_softmax_probs<1, false>, grid, block, 0, st, logits, rows, V, stride, Vu, G, k, T,
                          part, row_max, row_lse, probs);
}

}  // namespace specv
