// The verify window as a list of rows ("walk"), shared by the kernels that
// stream it: the row-statistics kernels and the top-p nucleus kernel.
//
// Request b owns (K+1) * l + bonus walk rows, l = its verify length: first
// its target rows 0..l-1 (plus target row l, the bonus row, when the walk
// includes it), then the K draft categories of l rows each. Every block
// builds the geometry in shared memory: rowoff[b] the first walk row of
// request b (rowoff[B] = total), base[b] the target row of its position 0.
#pragma once

#include "common.cuh"
#include "internal.h"

namespace specv {

struct Walk {
  const int* rowoff;
  const int* base;
};

// Row r of the walk and the address of the drafted token of its position
// (nullptr outside verify mode and for a bonus row). The token itself is
// loaded by the caller, which uses it only after the row's first data has
// arrived.
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
  const int l = (w.rowoff[b + 1] - w.rowoff[b] - rs.bonus) / (rs.K + 1);
  if (q < l + rs.bonus) {
    if (q < l) tokp = rs.tokens + static_cast<int64_t>(b) * rs.L + q;
    return static_cast<const char*>(rs.target) + (static_cast<int64_t>(w.base[b]) + q) * rs.stride * esz;
  }
  const int q2 = q - l - rs.bonus, z = q2 / l, i = q2 - z * l;
  tokp = rs.tokens + static_cast<int64_t>(b) * rs.L + i;
  return static_cast<const char*>(rs.draft) + ((static_cast<int64_t>(b) * rs.K + z) * rs.L + i) * rs.stride * esz;
}

__device__ __forceinline__ int load_token(const int32_t* tokp) { return tokp ? __ldg(tokp) : -1; }

// Rows of the walk; in verify mode also builds its geometry in shared memory
// (every thread of the block calls this).
template <int NT>
__device__ __forceinline__ int64_t build_walk(const RowSpace& rs, int* walk_smem, int* tmp) {
  if (!rs.verify) return rs.rows;
  int* rowoff = walk_smem;
  int* base = walk_smem + rs.B + 1;
  for (int b = threadIdx.x; b < rs.B; b += NT) {
    int l = rs.vlen ? rs.vlen[b] : rs.L;
    if (l < 0 || l > rs.L) l = 0;  // flagged by the sampling kernel
    rowoff[b] = (rs.K + 1) * l + rs.bonus;
    base[b] = rs.row_off ? rs.row_off[b] : b * (rs.L + 1);
  }
  __syncthreads();
  const int64_t nrows = block_exclusive_scan<NT>(rowoff, rs.B, tmp);
  if (threadIdx.x == 0) rowoff[rs.B] = static_cast<int>(nrows);
  __syncthreads();
  return nrows;
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

}  // namespace specv
