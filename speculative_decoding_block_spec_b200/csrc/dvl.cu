// Dynamic verify-length (DVL) allocation and packing.
//
// "DScale: Scaling Block-Diffusion Speculative Decoding with Adaptive
// Verification", Abstract: DVL allocation packs scored prefixes into half
// the native verification capacity, and fixed-address workspaces carry the
// changing boundaries through verification. Position i of request b is
// worth its prefix-survival probability P[b,i] = s[b,0] * ... * s[b,i] (the
// block-diffusion failure-mode Q&A: verify lengths from prefix survival
// probabilities). Each request keeps its root slot and the other slots go
// to the largest P overall, ordered (P desc, b asc, i asc); because each
// row's products are non-increasing the chosen set is a prefix of every row.
//
// k_dvl_allocate: one block per request. Every block forms all B*L products
// in shared memory (fp64, left to right), ranks its own L entries against
// all of them, and writes verify_len[b]. The last block (atomic ticket,
// reset by that block) scans the lengths into offsets and fills the slot
// map. k_dvl_pack then copies the selected dense target rows into the
// fixed-address packed buffer.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace specv {

constexpr int kDvlMaxL = 32;

__global__ void __launch_bounds__(kThreads) k_dvl_allocate(const float* __restrict__ scores, int B, int L,
                                                           int budget, int32_t* verify_len, int32_t* offsets,
                                                           int32_t* slot_map, int* status, int* ticket) {
  extern __shared__ double sP[];  // [B*L] products; reused as int[B+1] by the last block
  __shared__ int s_cnt[kDvlMaxL][kWarps];
  __shared__ int s_tmp[kWarps + 1];
  __shared__ int s_last;
  pdl_wait();
  pdl_trigger();
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int b = blockIdx.x;
  const int n = B * L;

  for (int r = tid; r < B; r += kThreads) {
    double P = 1.0;
    for (int i = 0; i < L; ++i) {
      P = P * static_cast<double>(scores[static_cast<int64_t>(r) * L + i]);
      sP[r * L + i] = P;
    }
  }
  if (tid < L) {
    const float s = scores[static_cast<int64_t>(b) * L + tid];
    if (!(s >= 0.f && s <= 1.f)) atomicOr(status, kFlagScores);
  }
  __syncthreads();

  const int64_t cap = static_cast<int64_t>(B) * (L + 1);
  const int take = static_cast<int>(std::min<int64_t>(budget, cap)) - B;
  // rank of (b, i) = number of entries ordered before it
  for (int i = 0; i < L; ++i) {
    const double Pi = sP[b * L + i];
    const int self = b * L + i;
    int c = 0;
    for (int e = tid; e < n; e += kThreads) {
      const double Pe = sP[e];
      c += (Pe > Pi || (Pe == Pi && e < self)) ? 1 : 0;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
    if (lane == 0) s_cnt[i][w] = c;
  }
  __syncthreads();
  if (tid < L) {
    int rank = 0;
    for (int k = 0; k < kWarps; ++k) rank += s_cnt[tid][k];
    s_cnt[tid][0] = rank < take ? 1 : 0;
  }
  __syncthreads();
  if (tid == 0) {
    int ell = 0;
    for (int i = 0; i < L; ++i) ell += s_cnt[i][0];
    verify_len[b] = ell;
    __threadfence();
    s_last = atomicAdd(ticket, 1) == B - 1;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();

  int* off = reinterpret_cast<int*>(sP);
  for (int r = tid; r < B; r += kThreads) off[r] = __ldcg(verify_len + r) + 1;
  __syncthreads();
  const int total = block_exclusive_scan(off, B, s_tmp);
  if (tid == 0) off[B] = total;
  __syncthreads();
  for (int r = tid; r <= B; r += kThreads) offsets[r] = off[r];
  if (slot_map) {
    for (int s = tid; s < budget; s += kThreads) {
      int v = -1;
      if (s < total) {
        int lo = 0, hi = B - 1;  // last request with off <= s
        while (lo < hi) {
          const int mid = (lo + hi + 1) >> 1;
          if (off[mid] <= s) lo = mid; else hi = mid - 1;
        }
        v = lo * (L + 1) + (s - off[lo]);
      }
      slot_map[s] = v;
    }
  }
  if (tid == 0) *ticket = 0;
}

// packed[offsets[b] + i] = dense[b, i] for i <= verify_len[b]; one block per
// (packed slot, chunk of the row).
template <bool VEC>
__global__ void __launch_bounds__(kThreads) k_dvl_pack(const char* __restrict__ dense, char* __restrict__ packed,
                                                       int64_t row_bytes, int B, int L, int64_t chunks,
                                                       const int32_t* __restrict__ offsets) {
  __shared__ int64_t s_src;
  pdl_wait();
  pdl_trigger();
  const int64_t slot = blockIdx.x / chunks, chunk = blockIdx.x % chunks;
  if (threadIdx.x == 0) {
    int64_t src = -1;
    if (slot < offsets[B]) {
      int lo = 0, hi = B - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (offsets[mid] <= slot) lo = mid; else hi = mid - 1;
      }
      src = static_cast<int64_t>(lo) * (L + 1) + (slot - offsets[lo]);
    }
    s_src = src;
  }
  __syncthreads();
  const int64_t src = s_src;
  if (src < 0) return;
  const char* s = dense + src * row_bytes;
  char* d = packed + slot * row_bytes;
  if constexpr (VEC) {
    const int64_t nv = row_bytes / 16;
    for (int64_t u = chunk * kThreads + threadIdx.x; u < nv; u += chunks * kThreads)
      reinterpret_cast<uint4*>(d)[u] = ldg16(reinterpret_cast<const uint4*>(s) + u);
  } else {
    for (int64_t u = chunk * kThreads + threadIdx.x; u < row_bytes; u += chunks * kThreads) d[u] = s[u];
  }
}

cudaError_t launch_dvl(const float* scores, int B, int L, int budget, int32_t* verify_len, int32_t* offsets,
                       int32_t* slot_map, int* status, int* ticket, cudaStream_t st) {
  const size_t smem = std::max(static_cast<size_t>(B) * L * sizeof(double), static_cast<size_t>(B + 1) * sizeof(int));
  if (smem > 48 * 1024) {
    const cudaError_t e =
        cudaFuncSetAttribute(k_dvl_allocate, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  return launch_pdl(k_dvl_allocate, dim3(B), dim3(kThreads), smem, st, scores, B, L, budget, verify_len, offsets,
                    slot_map, status, ticket);
}

cudaError_t launch_pack(const void* dense, void* packed, int dtype, int B, int L, int64_t V, int budget,
                        const int32_t* offsets, cudaStream_t st) {
  const int64_t row_bytes = V * (dtype == 0 ? 4 : 2);
  const bool vec = row_bytes % 16 == 0 && reinterpret_cast<uintptr_t>(dense) % 16 == 0 &&
                   reinterpret_cast<uintptr_t>(packed) % 16 == 0;
  const int64_t units = vec ? row_bytes / 16 : row_bytes;
  const int64_t per_block = static_cast<int64_t>(kThreads) * 4;
  const int64_t chunks = std::max<int64_t>(1, (units + per_block - 1) / per_block);
  const int64_t slots = std::min<int64_t>(budget, static_cast<int64_t>(B) * (L + 1));
  const dim3 grid(static_cast<unsigned>(slots * chunks));
  const char* d = static_cast<const char*>(dense);
  char* p = static_cast<char*>(packed);
  return vec ? launch_pdl(k_dvl_pack<true>, grid, dim3(kThreads), 0, st, d, p, row_bytes, B, L, chunks, offsets)
             : launch_pdl(k_dvl_pack<false>, grid, dim3(kThreads), 0, st, d, p, row_bytes, B, L, chunks, offsets);
}

}  // namespace specv
