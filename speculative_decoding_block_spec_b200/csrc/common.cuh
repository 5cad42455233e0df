// Device helpers shared by the specv kernels (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace specv {

constexpr int kThreads = 256;          // threads per block, every kernel
constexpr int kWarps = kThreads / 32;
constexpr int kGMax = 2048;            // upper bound on the row-statistics grid
constexpr int kPMax = 64;              // upper bound on blocks per request in the sampling kernel
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// Device status flags (mirror SPEC_DEV_* of the public header).
constexpr int kFlagTokenRange = 1;
constexpr int kFlagNonFinite = 2;
constexpr int kFlagVerifyLen = 4;
constexpr int kFlagScores = 8;

// ---------------------------------------------------------------- PTX wrappers

// Programmatic dependent launch: wait for the preceding grid's memory, and
// allow the next grid in the stream to be scheduled.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Hardware base-2 exponential / logarithm (MUFU), flush-to-zero.
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float lg2(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 16-byte streaming load through the read-only path, not kept in L1.
__device__ __forceinline__ uint4 ldg16(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// Packed bf16x2 maximum (exact; a NaN operand yields the other operand).
__device__ __forceinline__ uint32_t bmax2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Order key of a logit (bf16 logits widened exactly to fp32): the unsigned
// order of keys is the numeric order of the values, and equal values (+0 and
// -0 included) share one key.
__device__ __forceinline__ uint32_t order_key(float x) {
  uint32_t b = __float_as_uint(x);
  if (b == 0x80000000u) b = 0u;
  return (b >> 31) ? ~b : (b | 0x80000000u);
}

// ------------------------------------------------------------- element types

// Logit element types: fp32 (code 0) and bf16 (code 1, stored as uint16 bits).
template <int DT> struct Elem;
template <> struct Elem<0> {
  static constexpr int kBytes = 4;
  static constexpr int kPerVec = 4;  // elements per 16-byte vector
  __device__ __forceinline__ static float at(const void* row, int64_t v) {
    return __ldg(reinterpret_cast<const float*>(row) + v);
  }
  __device__ __forceinline__ static void unpack(const uint4& w, float (&x)[4]) {
    x[0] = __uint_as_float(w.x); x[1] = __uint_as_float(w.y);
    x[2] = __uint_as_float(w.z); x[3] = __uint_as_float(w.w);
  }
};
template <> struct Elem<1> {
  static constexpr int kBytes = 2;
  static constexpr int kPerVec = 8;
  __device__ __forceinline__ static float at(const void* row, int64_t v) {
    const unsigned short h = __ldg(reinterpret_cast<const unsigned short*>(row) + v);
    return __uint_as_float(static_cast<uint32_t>(h) << 16);
  }
  __device__ __forceinline__ static void unpack(const uint4& w, float (&x)[8]) {
    x[0] = bf16lo(w.x); x[1] = bf16hi(w.x); x[2] = bf16lo(w.y); x[3] = bf16hi(w.y);
    x[4] = bf16lo(w.z); x[5] = bf16hi(w.z); x[6] = bf16lo(w.w); x[7] = bf16hi(w.w);
  }
};

// ------------------------------------------------- online softmax statistics

// A partial softmax normaliser of raw logits: m = max x, s = sum 2^((x - m) k),
// k = log2(e) / T, so that log sum exp(x / T) = m / T + ln s.
//
// Merge (m2, s2) into (m, s). Symmetric: both argument orders round alike.
__device__ __forceinline__ void ms_merge(float& m, float& s, float m2, float s2, float k) {
  if (m2 > m) {
    s = fmaf(s, ex2((m - m2) * k), s2);
    m = m2;
  } else if (m2 == m) {
    s = s + s2;
  } else {
    s = fmaf(s2, ex2((m2 - m) * k), s);
  }
}

// Block-wide merge; the result is valid in every thread of warp 0.
__device__ __forceinline__ void block_merge(float& m, float& s, float k, float2* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
    const float s2 = __shfl_xor_sync(0xffffffffu, s, o);
    ms_merge(m, s, m2, s2, k);
  }
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[w] = make_float2(m, s);
  __syncthreads();
  if (w == 0) {
    float2 v = lane < kWarps ? red[lane] : make_float2(-INFINITY, 0.f);
    m = v.x;
    s = v.y;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
      const float s2 = __shfl_xor_sync(0xffffffffu, s, o);
      ms_merge(m, s, m2, s2, k);
    }
  }
  __syncthreads();
}

// ------------------------------------------------------------ work partition

// The row-statistics grid splits N work units evenly over G blocks: block c
// owns units [floor(c N / G), floor((c+1) N / G)). owner(e) is the block
// whose range holds unit e; the partial of (row r, block c) lives in slot
// c + r, which is unique because consecutive rows share at most their
// boundary block.
__host__ __device__ __forceinline__ int64_t split_start(int64_t c, int64_t N, int64_t G) {
  return c * N / G;
}
__host__ __device__ __forceinline__ int64_t split_owner(int64_t e, int64_t N, int64_t G) {
  return ((e + 1) * G - 1) / N;
}

// Exclusive scan over n small integers in shared memory, in place:
// arr[i] <- sum_{k<i} arr[k]; returns the total (to every thread). NT is the
// block size; `tmp` holds NT/32 + 1 ints. Must be called by the whole block.
template <int NT = kThreads>
__device__ __forceinline__ int block_exclusive_scan(int* arr, int n, int* tmp) {
  constexpr int NW = NT / 32;
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int per = (n + NT - 1) / NT;
  const int lo = min(n, tid * per), hi = min(n, lo + per);
  int local = 0;
  for (int i = lo; i < hi; ++i) local += arr[i];
  int incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) tmp[w] = incl;
  __syncthreads();
  if (tid == 0) {
    int run = 0;
    for (int k = 0; k < NW; ++k) {
      const int t = tmp[k];
      tmp[k] = run;
      run += t;
    }
    tmp[NW] = run;
  }
  __syncthreads();
  int run = tmp[w] + incl - local;
  for (int i = lo; i < hi; ++i) {
    const int t = arr[i];
    arr[i] = run;
    run += t;
  }
  const int total = tmp[NW];
  __syncthreads();
  return total;
}

// Fold N 16-byte vectors into the running (m, s): the group maximum exactly
// (raw bf16 pairs), a rescale of s when it grows, then one base-2
// exponential per element.
template <int DT, int N>
__device__ __forceinline__ void fold_vectors(const uint4 (&v)[N], float& m, float& s, float k) {
  constexpr int E = Elem<DT>::kPerVec;
  float gm;
  if constexpr (DT == 1) {
    uint32_t mx = bmax2(v[0].x, v[0].y);
    mx = bmax2(mx, bmax2(v[0].z, v[0].w));
#pragma unroll
    for (int t = 1; t < N; ++t) mx = bmax2(mx, bmax2(bmax2(v[t].x, v[t].y), bmax2(v[t].z, v[t].w)));
    gm = fmaxf(bf16lo(mx), bf16hi(mx));
  } else {
    gm = -INFINITY;
#pragma unroll
    for (int t = 0; t < N; ++t) {
      gm = fmaxf(gm, fmaxf(fmaxf(__uint_as_float(v[t].x), __uint_as_float(v[t].y)),
                           fmaxf(__uint_as_float(v[t].z), __uint_as_float(v[t].w))));
    }
  }
  if (gm > m) {
    s *= ex2((m - gm) * k);
    m = gm;
  }
  if (m == -INFINITY) return;  // every element so far is -inf: nothing to add
  float part[N];
#pragma unroll
  for (int t = 0; t < N; ++t) {
    float x[E];
    Elem<DT>::unpack(v[t], x);
    float e[E];
#pragma unroll
    for (int i = 0; i < E; ++i) e[i] = ex2((x[i] - m) * k);
#pragma unroll
    for (int w = 1; w < E; w <<= 1)
#pragma unroll
      for (int i = 0; i < E; i += 2 * w) e[i] += e[i + w];
    part[t] = e[0];
  }
#pragma unroll
  for (int w = 1; w < N; w <<= 1)
#pragma unroll
    for (int i = 0; i + w < N; i += 2 * w) part[i] += part[i + w];
  s += part[0];
}

}  // namespace specv
