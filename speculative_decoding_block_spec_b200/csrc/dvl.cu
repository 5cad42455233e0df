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
// k_dvl_allocate: one block of 1024 threads does the whole allocation, in
// shared memory, with no cross-block hand-off:
//  1. one thread per request forms its products in fp64, left to right, and
//     stores them as 64-bit keys whose unsigned order is the order of P
//     (+0 and -0 are one key, as they compare equal);
//  2. a radix select over the keys, 8-bit digits from the highest bit on
//     which two keys differ, finds the cut: per digit a 256-bin histogram of
//     the entries that still match the prefix (one shared atomic per entry;
//     starting below the common bits spreads the first digit over many bins)
//     and one warp's suffix scan over it; the descent stops at the first digit
//     whose bin is taken whole; entries above the cut are selected, and of
//     those equal to it the first ones by flat index (a block scan of the
//     equal entries' flags);
//  3. verify_len[b] = selected entries of row b; an exclusive scan of
//     verify_len + 1 gives the offsets, from which the slot map is filled.
// k_dvl_pack then copies the selected dense target rows into the
// fixed-address packed buffer.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace specv {

#ifndef SPECV_DVL_THREADS
#define SPECV_DVL_THREADS 1024
#endif
constexpr int kDvlThreads = SPECV_DVL_THREADS;  // one block; 256 ... 1024 threads
constexpr int kDvlWarps = kDvlThreads / 32;
constexpr int kDvlMaxL = 32;  // SPEC_MAX_L

// Order-preserving key of a product: unsigned order of the key = numeric
// order of P (negative values below +0; -0 maps to the key of +0; a NaN,
// possible only from a flagged score, lands at one end).
__device__ __forceinline__ unsigned long long p_key(double P) {
  if (P == 0.0) P = 0.0;
  const unsigned long long b = static_cast<unsigned long long>(__double_as_longlong(P));
  return (b >> 63) ? ~b : (b | (1ull << 63));
}

// offsets[0..B] from the scanned lengths `off` (off[B] = total), and the slot
// map: slot s -> b * (L + 1) + (s - off[b]) for the request b holding it, -1
// past the total. Called by the whole block.
__device__ __forceinline__ void write_offsets_and_slots(const int* off, int B, int L, int budget, int total,
                                                        int32_t* offsets, int32_t* slot_map) {
  for (int r = threadIdx.x; r <= B; r += kDvlThreads) offsets[r] = off[r];
  if (!slot_map) return;
  for (int s = threadIdx.x; s < budget; s += kDvlThreads) {
    int v = -1;
    if (s < total) {
      int lo = 0, hi = B - 1;  // last request with offset <= s
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (off[mid] <= s) lo = mid; else hi = mid - 1;
      }
      v = lo * (L + 1) + (s - off[lo]);
    }
    slot_map[s] = v;
  }
}

__global__ void __launch_bounds__(kDvlThreads, 1) k_dvl_allocate(const float* __restrict__ scores, int B, int L,
                                                               int budget, int32_t* verify_len, int32_t* offsets,
                                                               int32_t* slot_map, int* status) {
  extern __shared__ unsigned long long sKey[];  // [B*L] keys, then int[B*L] equal-key ranks, int[B + 1] lengths
  __shared__ int s_hist[256];
  __shared__ int s_tmp[kDvlWarps + 1];
  __shared__ int s_digit, s_k, s_binc, s_flag;
  __shared__ unsigned long long s_or, s_and;
  pdl_wait();
  pdl_trigger();
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int n = B * L;
  int* sRank = reinterpret_cast<int*>(sKey + n);  // index-order rank among the entries equal to the cut key
  int* lens = sRank + n;                           // verify_len + 1, then offsets

  if (tid == 0) {
    s_flag = 0;
    s_or = 0ull;
    s_and = ~0ull;
  }
  for (int r = tid; r < B; r += kDvlThreads) lens[r] = 0;  // past the staged scores
  int bad = 0;
  unsigned long long kor = 0ull, kand = ~0ull;  // OR and AND of this thread's keys (the radix descent's start)
  if (L % 4 == 0 && L <= kDvlMaxL && (reinterpret_cast<uintptr_t>(scores) & 15) == 0) {
    // a thread's row as 16-byte vectors straight into registers (one memory round trip), then the products
    __syncthreads();  // s_or / s_and initialised
    for (int r = tid; r < B; r += kDvlThreads) {
      float4 v[kDvlMaxL / 4];
#pragma unroll
      for (int q = 0; q < kDvlMaxL / 4; ++q)
        if (q < L / 4) v[q] = __ldg(reinterpret_cast<const float4*>(scores + static_cast<int64_t>(r) * L) + q);
      double P = 1.0;
#pragma unroll
      for (int q = 0; q < kDvlMaxL / 4; ++q) {
        if (q < L / 4) {
          const float sv[4] = {v[q].x, v[q].y, v[q].z, v[q].w};
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            bad |= !(sv[c] >= 0.f && sv[c] <= 1.f);
            P = P * static_cast<double>(sv[c]);
            const unsigned long long key = p_key(P);
            sKey[r * L + 4 * q + c] = key;
            kor |= key;
            kand &= key;
          }
        }
      }
    }
  } else {
    __syncthreads();  // s_or / s_and initialised
    float* stage = reinterpret_cast<float*>(sKey + n);  // the scores, loaded coalesced (space reused below)
    for (int e = tid; e < n; e += kDvlThreads) stage[e] = scores[e];
    __syncthreads();
    for (int r = tid; r < B; r += kDvlThreads) {
      double P = 1.0;
      for (int i = 0; i < L; ++i) {
        const float sv = stage[r * L + i];
        bad |= !(sv >= 0.f && sv <= 1.f);
        P = P * static_cast<double>(sv);
        const unsigned long long key = p_key(P);
        sKey[r * L + i] = key;
        kor |= key;
        kand &= key;
      }
    }
  }
  {  // the bits above the highest one on which two keys differ are common to all (used by the radix descent)
    const unsigned ohi = __reduce_or_sync(0xffffffffu, static_cast<unsigned>(kor >> 32));
    const unsigned olo = __reduce_or_sync(0xffffffffu, static_cast<unsigned>(kor));
    const unsigned ahi = __reduce_and_sync(0xffffffffu, static_cast<unsigned>(kand >> 32));
    const unsigned alo = __reduce_and_sync(0xffffffffu, static_cast<unsigned>(kand));
    if (lane == 0) {
      atomicOr(&s_or, (static_cast<unsigned long long>(ohi) << 32) | olo);
      atomicAnd(&s_and, (static_cast<unsigned long long>(ahi) << 32) | alo);
    }
  }
  if (bad) atomicOr(&s_flag, kFlagScores);
  __syncthreads();

  const int64_t cap = static_cast<int64_t>(B) * (L + 1);
  const int take = static_cast<int>(std::min<int64_t>(budget, cap)) - B;  // 0 <= take <= n
  // The cut: entries whose key, under `mask`, is above `prefix` are selected; of those equal to it under the
  // mask, all are selected when the bin holds exactly the k still wanted, else (equal full keys) the first k
  // by flat index. take == 0 selects nothing: no masked key exceeds the all-ones prefix.
  unsigned long long prefix = ~0ull, mask = ~0ull;
  int k = 0, binc = 0;
  if (take > 0) {
    // the bits above the highest one on which two keys differ are common to all: the descent starts below
    // them (products in [0, 1] share the sign and most exponent bits, a whole digit or more)
    const unsigned long long diff = s_or ^ s_and;
    k = take;  // rank (1-based, descending) of the wanted entry among those matching the prefix
    if (diff == 0ull) {  // one key: the cut is that key, taken by flat index
      prefix = s_and;
      binc = n;
    } else {
      const int hb = 63 - __clzll(static_cast<long long>(diff));
      mask = hb == 63 ? 0ull : ~((2ull << hb) - 1ull);
      prefix = s_and & mask;
    }
    for (int shift = max(0, (diff == 0ull ? 0 : 63 - __clzll(static_cast<long long>(diff))) - 7);
         diff != 0ull; shift = max(0, shift - 8)) {
      if (tid < 256) s_hist[tid] = 0;
      __syncthreads();
      for (int base = wid * 32; base < n; base += kDvlThreads) {
        const int e = base + lane;
        const unsigned long long u = e < n ? sKey[e] : 0ull;
        const int d = (e < n && (u & mask) == prefix) ? static_cast<int>((u >> shift) & 255) : 256;
        if (d < 256) atomicAdd(&s_hist[d], 1);
      }
      __syncthreads();
      if (wid == 0) {  // lane l owns digits 255 - 8l ... 248 - 8l (descending)
        int c[8], sum = 0;
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          c[t] = s_hist[255 - 8 * lane - t];
          sum += c[t];
        }
        int incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int v = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += v;
        }
        const int excl = incl - sum;
        if (excl < k && incl >= k) {  // the wanted entry's digit is in this lane's range
          int run = excl;
#pragma unroll
          for (int t = 0; t < 8; ++t) {
            if (run < k && run + c[t] >= k) {
              s_digit = 255 - 8 * lane - t;
              s_k = k - run;
              s_binc = c[t];
            }
            run += c[t];
          }
        }
      }
      __syncthreads();
      // s_digit, s_k and s_binc are rewritten only after two more barriers of the next digit
      prefix |= static_cast<unsigned long long>(s_digit) << shift;
      mask |= 255ull << shift;
      k = s_k;
      binc = s_binc;
      if (binc == k || shift == 0) break;  // the whole bin is taken, or every bit decided (block-uniform)
    }
  }

  // entries equal to the cut under the mask: all taken, or (ties of full keys) the first k by flat index
  const bool rank_eq = take > 0 && binc > k;
  if (rank_eq) {
    for (int e = tid; e < n; e += kDvlThreads) sRank[e] = (sKey[e] & mask) == prefix;
    __syncthreads();
    block_exclusive_scan<kDvlThreads>(sRank, n, s_tmp);
  }
  // verify_len[b]: selected entries of row b (a prefix of the row when every score is in [0, 1]), one thread
  // per entry
  for (int e = tid; e < n; e += kDvlThreads) {
    const unsigned long long um = sKey[e] & mask;
    if (um > prefix || (um == prefix && take > 0 && (rank_eq ? sRank[e] < k : true))) atomicAdd(&lens[e / L], 1);
  }
  __syncthreads();
  for (int r = tid; r < B; r += kDvlThreads) {
    const int ell = lens[r];
    verify_len[r] = ell;
    lens[r] = ell + 1;
  }
  __syncthreads();
  const int total = block_exclusive_scan<kDvlThreads>(lens, B, s_tmp);
  if (tid == 0) lens[B] = total;
  __syncthreads();
  write_offsets_and_slots(lens, B, L, budget, total, offsets, slot_map);
  if (tid == 0 && s_flag) atomicOr(status, s_flag);
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
                       int32_t* slot_map, int* status, cudaStream_t st) {
  const int64_t n = static_cast<int64_t>(B) * L;
  // keys, equal-key ranks, lengths
  const size_t smem = static_cast<size_t>(n) * (sizeof(unsigned long long) + sizeof(int)) +
                      static_cast<size_t>(B + 1) * sizeof(int);
  if (smem > 48 * 1024) {
    const cudaError_t e =
        cudaFuncSetAttribute(k_dvl_allocate, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  return launch_pdl(k_dvl_allocate, dim3(1), dim3(kDvlThreads), smem, st, scores, B, L, budget, verify_len, offsets,
                    slot_map, status);
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
