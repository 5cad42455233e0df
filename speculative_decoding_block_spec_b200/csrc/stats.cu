// Row statistics of temperature softmax (the bandwidth-bound hot loop) and
// the finalisation used by spec_softmax_T.
//
// Temperature softmax of target and draft logit rows, z = x / T: the
// verifier samples both with one sampling filter ("DBLAST: Dependent Block
// Drafting for Stochastic Speculative Decoding", Pith review, "Assumptions";
// target sampling at T = 1.5 in "What would settle it").
//
// Design. A grid of G blocks splits the flattened 16-byte units of every row
// evenly, so every block streams the same number of bytes whatever the row
// count; a block's range covers a tail of one row, whole rows, and a head of
// another. Each thread keeps an online (max, sum of 2^((x - max) log2e / T))
// over its vectors: a group is loaded at once, its maximum taken exactly on
// the raw bf16 pairs, then one exponential per element. Blocks write one
// partial per (row, block); consumers merge the few partials of a row. Two
// kernels share this split: k_row_stats (several blocks per SM, each thread
// striding its block's range) and k_row_stats_dyn (one block per SM whose
// warps take row-aligned slices of the range from a shared counter, for
// windows of at most 256 MB).
#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "walk.cuh"

namespace specv {

constexpr int kUnroll = 4;  // 16-byte vectors in flight per thread per group

// Vector path: each segment (the block's part of one row) streams groups of
// kUnroll 16-byte vectors per thread, then single vectors, and ends with one
// block merge. The drafted token is loaded with the row's first data; after
// the segment, the thread whose units hold it re-reads that element (the row
// has just passed through L2) and stores it once the merge is done, so
// neither load stalls the stream.
template <int DT>
__device__ __forceinline__ void walk_vec(const RowSpace& rs, const Walk& w, int64_t Vu, int64_t e0, int64_t e1,
                                         float k, float2* __restrict__ part, float2* red) {
  constexpr int E = Elem<DT>::kPerVec;
  const int tid = threadIdx.x;
  for (int64_t e = e0; e < e1;) {
    const int64_t r = e / Vu;
    const int u0 = static_cast<int>(e - r * Vu), u1 = static_cast<int>(min(e1, (r + 1) * Vu) - r * Vu);
    const int32_t* tokp;
    const char* row = locate<DT>(rs, w, r, tokp);
    const uint4* rv = reinterpret_cast<const uint4*>(row);
    const int tok = load_token(tokp);
    float m = -INFINITY, s = 0.f;
    int u = u0 + tid;
    for (; u + (kUnroll - 1) * kThreads < u1; u += kUnroll * kThreads) {
      uint4 v[kUnroll];
#pragma unroll
      for (int t = 0; t < kUnroll; ++t) v[t] = ldg16(rv + u + t * kThreads);
      fold_vectors<DT, kUnroll>(v, m, s, k);
    }
    for (; u < u1; u += kThreads) {
      const uint4 v[1] = {ldg16(rv + u)};
      fold_vectors<DT, 1>(v, m, s, k);
    }
    const int tu = tok / E;  // tok < 0: no token; tok >= V: matches no unit
    const bool hit = tok >= 0 && tu >= u0 && tu < u1 && (tu - u0) % kThreads == tid;
    const float xv = hit ? Elem<DT>::at(row, tok) : 0.f;
    block_merge(m, s, k, red);
    if (tid == 0) part[blockIdx.x + r] = make_float2(m, s);
    if (hit) rs.xg[r] = xv;
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
  const Walk w{walk_smem, walk_smem + rs.B + 1};
  const int64_t N = build_walk<kThreads>(rs, walk_smem, tmp) * Vu;
  const int64_t e0 = split_start(blockIdx.x, N, G), e1 = split_start(blockIdx.x + 1, N, G);
  if (e0 >= e1) return;  // empty share (N < grid): no partials
  if constexpr (VEC) walk_vec<DT>(rs, w, Vu, e0, e1, k, part, red);
  else walk_scalar<DT>(rs, w, Vu, e0, e1, k, part, red);
}

// ------------------------------------------------ balanced vector kernel
//
// One block of kDynThreads per SM, each block with an even share of the
// flattened units as above. Inside the block the share is cut into slices of
// kSlice units that never cross a row (a row's piece of the share is a
// segment); warps take slices in order from a shared-memory counter, with
// the next slice's loads in flight while the current one is folded, so every
// warp of an SM streams until the share is exhausted and the block ends
// within about one slice of its fastest warp. A warp folds the slices of one
// segment into its own (max, sum); when it moves on it stores that pair in
// a [warp][segment] table, and the block merges each segment's column into
// the (block, row) partial at the end. Used when a share spans at most
// kMaxSegs rows.
constexpr int kDynThreads = 1024;
constexpr int kDynWarps = kDynThreads / 32;
constexpr int kMaxSegs = 32;
constexpr int kSliceVec = 4;              // 16-byte vectors per lane per slice
constexpr int kSlice = 32 * kSliceVec;    // units per slice

__device__ __forceinline__ void warp_merge(float& m, float& s, float k) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
    const float s2 = __shfl_xor_sync(0xffffffffu, s, o);
    ms_merge(m, s, m2, s2, k);
  }
}

// Lane's vectors of slice position g (row-relative unit of lane 0), -inf past `end`.
template <int DT>
__device__ __forceinline__ void load_slice(const char* row, int g, int end, uint4 (&v)[kSliceVec]) {
  const uint4* rv = reinterpret_cast<const uint4*>(row);
  const uint32_t ninf = DT == 1 ? 0xFF80FF80u : 0xFF800000u;  // four or eight -inf: add nothing
#pragma unroll
  for (int t = 0; t < kSliceVec; ++t) {
    const int u = g + t * 32;
    v[t] = u < end ? ldg16(rv + u) : make_uint4(ninf, ninf, ninf, ninf);
  }
}

template <int DT>
__global__ void __launch_bounds__(kDynThreads, 1) k_row_stats_dyn(RowSpace rs, int64_t Vu, int G, float k,
                                                                  float2* __restrict__ part) {
  constexpr int E = Elem<DT>::kPerVec;
  extern __shared__ int walk_smem[];  // verify mode: rowoff[B + 1], base[B]
  __shared__ float2 s_tab[kDynWarps][kMaxSegs];
  __shared__ const char* s_ptr[kMaxSegs];
  __shared__ const int32_t* s_tokp[kMaxSegs];
  __shared__ int s_a[kMaxSegs], s_b[kMaxSegs], s_first[kMaxSegs + 1];
  __shared__ int s_next;
  __shared__ int tmp[kDynWarps + 1];
  pdl_wait();
  pdl_trigger();
  const Walk w{walk_smem, walk_smem + rs.B + 1};
  const int64_t N = build_walk<kDynThreads>(rs, walk_smem, tmp) * Vu;
  const int64_t e0 = split_start(blockIdx.x, N, G), e1 = split_start(blockIdx.x + 1, N, G);
  if (e0 >= e1) return;  // empty share (N < grid): no partials
  const int64_t r0 = e0 / Vu;
  const int nseg = static_cast<int>((e1 - 1) / Vu - r0 + 1);
  if (nseg > kMaxSegs) return;  // excluded by the host's choice of kernel
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  if (tid < nseg) {
    const int64_t r = r0 + tid;
    s_a[tid] = static_cast<int>(max(e0, r * Vu) - r * Vu);
    s_b[tid] = static_cast<int>(min(e1, (r + 1) * Vu) - r * Vu);
    const int32_t* tp;
    s_ptr[tid] = locate<DT>(rs, w, r, tp);
    s_tokp[tid] = tp;
  }
  for (int i = tid; i < kDynWarps * kMaxSegs; i += kDynThreads) (&s_tab[0][0])[i] = make_float2(-INFINITY, 0.f);
  if (tid == 0) s_next = 0;
  __syncthreads();
  if (tid < 32) {  // first slice of each segment (inclusive scan of slice counts)
    int n = lane < nseg ? (s_b[lane] - s_a[lane] + kSlice - 1) / kSlice : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, n, o);
      if (lane >= o) n += t;
    }
    s_first[lane + 1] = n;
    if (lane == 0) s_first[0] = 0;
  }
  __syncthreads();
  const int nslices = s_first[nseg];

  // The last warp first records the drafted-token logit of every segment whose
  // token falls in this block's share (two dependent loads), then joins the
  // stream late; the other warps take the slices it does not.
  if (wid == kDynWarps - 1 && lane < nseg) {
    const int tok = load_token(s_tokp[lane]);
    if (tok >= 0 && tok / E >= s_a[lane] && tok / E < s_b[lane]) rs.xg[r0 + lane] = Elem<DT>::at(s_ptr[lane], tok);
  }

  int seg = 0;  // this warp's segment cursor (slices are taken in increasing order)
  int kc;
  if (lane == 0) kc = atomicAdd(&s_next, 1);
  kc = __shfl_sync(0xffffffffu, kc, 0);
  uint4 vc[kSliceVec];
  int segc = 0, gc = 0;
  if (kc < nslices) {
    while (s_first[seg + 1] <= kc) ++seg;
    segc = seg;
    gc = s_a[seg] + (kc - s_first[seg]) * kSlice + lane;
    load_slice<DT>(s_ptr[seg], gc, s_b[seg], vc);
  }
  float m = -INFINITY, s = 0.f;
  int acc = segc;
  while (kc < nslices) {
    int kn;
    if (lane == 0) kn = atomicAdd(&s_next, 1);
    kn = __shfl_sync(0xffffffffu, kn, 0);
    uint4 vn[kSliceVec];
    int segn = segc, gn = 0;
    if (kn < nslices) {  // the next slice's loads go out before this one is folded
      while (s_first[seg + 1] <= kn) ++seg;
      segn = seg;
      gn = s_a[seg] + (kn - s_first[seg]) * kSlice + lane;
      load_slice<DT>(s_ptr[seg], gn, s_b[seg], vn);
    }
    if (segc != acc) {  // this warp is done with segment acc
      warp_merge(m, s, k);
      if (lane == 0) s_tab[wid][acc] = make_float2(m, s);
      m = -INFINITY;
      s = 0.f;
      acc = segc;
    }
    fold_vectors<DT, kSliceVec>(vc, m, s, k);
#pragma unroll
    for (int t = 0; t < kSliceVec; ++t) vc[t] = vn[t];
    kc = kn;
    segc = segn;
    gc = gn;
  }
  warp_merge(m, s, k);
  if (lane == 0) s_tab[wid][acc] = make_float2(m, s);  // (-inf, 0) if this warp had no slice
  __syncthreads();
  for (int sg = wid; sg < nseg; sg += kDynWarps) {
    float2 v = s_tab[lane][sg];
    warp_merge(v.x, v.y, k);
    if (lane == 0) part[blockIdx.x + r0 + sg] = v;
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

static int device_sms() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  static std::mutex mu;
  static int cache[64] = {0};
  std::lock_guard<std::mutex> lock(mu);
  if (dev < 64 && cache[dev]) return cache[dev];
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1) sms = 148;
  if (dev < 64) cache[dev] = sms;
  return sms;
}

// The balanced kernel runs one block per SM; it needs 16-byte vectors, a
// share of at most kMaxSegs rows per block and at least one slice per warp.
// It is chosen for windows of at most kDynMaxBytes: there the tail of
// unevenly progressing blocks is a large part of the launch, and on B200 it
// measured faster than the even split (78 MB: 21.5 against 23.0 us; 146 MB:
// equal), while on windows of 0.7-0.8 GB the even split was as fast or faster.
constexpr int64_t kDynMaxBytes = int64_t{256} << 20;

static bool use_dyn(bool vec, int64_t max_units, int64_t Vu, int G) {
  if (!vec || G != device_sms() || max_units * 16 > kDynMaxBytes) return false;
  const int64_t share = (max_units + G - 1) / G;
  return share >= static_cast<int64_t>(kDynThreads / 32) * kSlice && (share + Vu - 1) / Vu + 1 <= kMaxSegs;
}

int stats_grid(int dtype, bool vec, int64_t max_units, int64_t Vu) {
  if (use_dyn(vec, max_units, Vu, device_sms())) return device_sms();
  int g;
  if (dtype == 0) g = vec ? occupancy_of<0, true>() : occupancy_of<0, false>();
  else g = vec ? occupancy_of<1, true>() : occupancy_of<1, false>();
  // at least one unit per thread, and up to one block per row: a small window's rows are then streamed in
  // parallel rather than one after another by a single block
  const int64_t need = std::max<int64_t>((max_units + kThreads - 1) / kThreads, (max_units + Vu - 1) / Vu);
  return static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(g, need)));
}

cudaError_t launch_row_stats(const RowSpace& rs, int dtype, bool vec, int64_t V, float T, int G, float2* part,
                             cudaStream_t st) {
  const int64_t Vu = units_per_row(V, dtype, vec);
  const float k = log2e_over(T);
  const size_t smem = rs.verify ? static_cast<size_t>(2 * rs.B + 1) * sizeof(int) : 0;
  const dim3 grid(G), block(kThreads);
  const int64_t max_units =
      (rs.verify ? static_cast<int64_t>(rs.B) * ((rs.K + 1) * rs.L + rs.bonus) : rs.rows) * Vu;
  if (use_dyn(vec, max_units, Vu, G))
    return dtype == 0 ? launch_pdl(k_row_stats_dyn<0>, grid, dim3(kDynThreads), smem, st, rs, Vu, G, k, part)
                      : launch_pdl(k_row_stats_dyn<1>, grid, dim3(kDynThreads), smem, st, rs, Vu, G, k, part);
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
