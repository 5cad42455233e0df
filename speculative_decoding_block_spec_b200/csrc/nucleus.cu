// Top-p (nucleus) filtering of every row of the verify window, and the row
// statistics the filtered verification needs.
//
// Target sampling with a temperature and a top-p filter, target
// probabilities taken under the same sampling filter ("DBLAST: Dependent
// Block Drafting for Stochastic Speculative Decoding", Pith review, "What
// would settle it": T = 1.5, top-p 0.95; "Assumptions"). The filter of a row
// keeps its nucleus: the shortest run of tokens, in the order (probability
// descending, index ascending), whose mass reaches top_p; the kept tokens
// are renormalised and every other token gets probability 0. The same filter
// applies to the target rows and to every draft category.
//
// Probability is monotone in the logit, so the order is that of the logits,
// and the nucleus is fixed by a cut: the logit value x_c and token v_c of its
// last member; token v is kept iff x_v > x_c, or x_v == x_c and v <= v_c.
//
// k_nucleus, one row at a time per block (one block per SM, rows strided over
// the grid), in place of the statistics kernel when rows are filtered:
//  bf16 rows: one HBM pass counts the tokens of every bf16 bit pattern
//    (65,536 16-bit counters packed two to a 32-bit word in shared memory,
//    native integer atomics; -0 counted as +0) and records the drafted
//    token's logit. Everything else follows from the counts: the row
//    maximum m is the largest value present (a NaN or +inf present, or only
//    -inf, marks the row non-finite); the warps walk the values from the
//    largest down, each value's mass being its count times round(2^((x - m)
//    k) 2^42), in exact integers: the total is the normaliser, and the value
//    whose mass carries the running total across top_p * total is the cut.
//    A row whose counters could have wrapped (their total is not V) takes
//    the fp32 route below.
//  fp32 rows: a pass for the maximum and the drafted token's logit, then a
//    radix descent over 32-bit order keys: per digit (bits 31..20, 19..8,
//    7..0) the fixed-point mass of the tokens matching the prefix found so
//    far, with 64-bit integer atomics, and a descending scan for the digit
//    where the running mass crosses top_p * total.
//  Then the tokens of the cut value needed, n; if not all of them, the n-th
//  in index order is found with a warp-ordered count (the tie cut), which
//  re-reads the row from L2. Outputs per row: m, the log of the nucleus mass
//  sum_{v kept} 2^((x_v - m) k) (the filtered normaliser), the cut key, the
//  cut token and the drafted token's logit.
#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "walk.cuh"

namespace specv {

constexpr int kNucThreads = 1024;
constexpr int kNucWarps = kNucThreads / 32;
constexpr int kFix = 42;              // fixed-point scale of the masses: sums of up to 2^20 terms of <= 1 fit 2^62
constexpr int kNucBins = 4096;        // bins of the widest radix digit
constexpr int kValueWords = 32768;    // bf16: 65,536 16-bit counters, two per word
constexpr int kNucCountBins = 256;    // bins of the last digit, which also counts tokens

// round(q * 2^kFix) for q in [0, 1] (fp32 bits; no conversion instruction).
__device__ __forceinline__ unsigned long long to_fixed(float q) {
  const uint32_t b = __float_as_uint(q);
  const int e = static_cast<int>(b >> 23);
  if (e == 0) return 0ull;
  const uint32_t mant = (b & 0x7FFFFFu) | 0x800000u;  // q = mant * 2^(e - 150)
  const int sh = e - 150 + kFix;
  if (sh >= 0) return static_cast<unsigned long long>(mant) << sh;
  if (sh <= -25) return 0ull;                          // below half a unit
  return static_cast<unsigned long long>((mant + (1u << (-sh - 1))) >> (-sh));
}

// Block-wide exclusive scan of one value per thread (thread order), for a
// block of NT threads; `tmp` holds NT / 32 + 1 values. Returns the exclusive
// prefix.
template <typename T, int NT>
__device__ __forceinline__ T block_scan(T v, T* tmp) {
  constexpr int NW = NT / 32;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  T incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const T t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) tmp[w] = incl;
  __syncthreads();
  if (threadIdx.x == 0) {
    T run = 0;
    for (int k = 0; k < NW; ++k) {
      const T t = tmp[k];
      tmp[k] = run;
      run += t;
    }
    tmp[NW] = run;
  }
  __syncthreads();
  const T excl = tmp[w] + incl - v;
  __syncthreads();
  return excl;
}

__device__ __forceinline__ unsigned long long block_scan_u64(unsigned long long v, unsigned long long* tmp) {
  return block_scan<unsigned long long, kNucThreads>(v, tmp);
}

// One digit of the descent: hist[d] += fixed mass of every token whose key
// matches `prefix` under `pmask`, d = (key >> shift) & dmask; with `count`
// also cnt[d] += 1. Called by the whole block.
template <int DT, bool VEC>
__device__ __forceinline__ void digit_pass(const char* row, int64_t V, float m, float k, uint32_t prefix,
                                           uint32_t pmask, int shift, uint32_t dmask, bool count,
                                           unsigned long long* hist, unsigned* cnt) {
  constexpr int E = VEC ? Elem<DT>::kPerVec : 1;
  constexpr int U = VEC ? 2 : 1;  // units in flight per thread (the radix path is the rare one)
  const int64_t Vu = V / E;
  for (int64_t u0 = threadIdx.x; u0 < Vu; u0 += U * kNucThreads) {
    float x[U][E];
#pragma unroll
    for (int h = 0; h < U; ++h) {
      const int64_t u = u0 + static_cast<int64_t>(h) * kNucThreads;
      if (u >= Vu) break;
      if constexpr (VEC) Elem<DT>::unpack(ldg16(reinterpret_cast<const uint4*>(row) + u), x[h]);
      else x[h][0] = Elem<DT>::at(row, u);
    }
#pragma unroll
    for (int h = 0; h < U; ++h) {
      if (u0 + static_cast<int64_t>(h) * kNucThreads >= Vu) break;
#pragma unroll
      for (int e = 0; e < E; ++e) {
        const uint32_t key = order_key(x[h][e]);
        if ((key & pmask) != prefix) continue;
        const uint32_t d = (key >> shift) & dmask;
        const unsigned long long fx = to_fixed(ex2((x[h][e] - m) * k));
        if (fx) atomicAdd(&hist[d], fx);
        if (count) atomicAdd(&cnt[d], 1u);
      }
    }
  }
}

// The digit d, scanning bins nb-1 down to 0 from the running mass `above`,
// whose bin takes the running mass from below `target` to at least it; also
// the running mass above that bin. Called by the whole block.
__device__ __forceinline__ void find_digit(const unsigned long long* hist, int nb, unsigned long long above,
                                           unsigned long long target, unsigned long long* tmp, int* s_d,
                                           unsigned long long* s_above) {
  if (threadIdx.x == 0) {  // defaults, overwritten by the one thread whose bins hold the crossing
    *s_d = 0;
    *s_above = above;
  }
  const int per = (nb + kNucThreads - 1) / kNucThreads;
  const int hi = nb - 1 - threadIdx.x * per;  // this thread's bins: hi, hi - 1, ... (descending)
  unsigned long long local = 0;
  for (int t = 0; t < per; ++t)
    if (hi - t >= 0) local += hist[hi - t];
  unsigned long long run = above + block_scan_u64(local, tmp);
  for (int t = 0; t < per; ++t) {
    const int d = hi - t;
    if (d < 0) break;
    const unsigned long long h = hist[d];
    if (run < target && run + h >= target) {
      *s_d = d;
      *s_above = run;
    }
    run += h;
  }
  __syncthreads();
}

// Index (in row order) of the n-th token (1-based) whose key is kappa; the
// row holds at least n of them. Called by the whole block.
template <int DT, bool VEC, int NW = kNucWarps>
__device__ __forceinline__ int64_t nth_equal(const char* row, int64_t V, uint32_t kappa, unsigned n, unsigned* s_wc,
                                             long long* s_v) {
  constexpr int E = VEC ? Elem<DT>::kPerVec : 1;
  const int64_t Vu = V / E;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int64_t cw = (Vu + NW - 1) / NW;  // units per warp, contiguous
  const int64_t a = min(Vu, w * cw), b = min(Vu, a + cw);
  // bf16 vectors compare raw bit pairs: the raw bits of the cut value (and
  // those of -0 when the cut value is zero) in both halves of a word
  const uint32_t k16 = kappa >> 16;
  const uint32_t hraw = (k16 & 0x8000u) ? (k16 & 0x7FFFu) : (~k16 & 0xFFFFu);
  const uint32_t hh = hraw | (hraw << 16);
  const bool zero = hraw == 0u;
  auto matches = [&](int64_t u) -> unsigned {  // bit e set when element e of unit u has key kappa
    if constexpr (DT == 1 && VEC) {
      const uint4 q = ldg16(reinterpret_cast<const uint4*>(row) + u);
      const uint32_t ws[4] = {q.x, q.y, q.z, q.w};
      unsigned bits = 0;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t eq = __vcmpeq2(ws[c], hh);
        if (zero) eq |= __vcmpeq2(ws[c], 0x80008000u);
        bits |= ((eq & 1u) << (2 * c)) | (((eq >> 16) & 1u) << (2 * c + 1));
      }
      return bits;
    } else {
      float x[E];
      if constexpr (VEC) Elem<DT>::unpack(ldg16(reinterpret_cast<const uint4*>(row) + u), x);
      else x[0] = Elem<DT>::at(row, u);
      unsigned bits = 0;
#pragma unroll
      for (int e = 0; e < E; ++e) bits |= (order_key(x[e]) == kappa ? 1u : 0u) << e;
      return bits;
    }
  };
  if (threadIdx.x == 0) *s_v = V - 1;  // overwritten by the lane that finds the token
  unsigned c = 0;
  for (int64_t u = a + lane; u < b; u += 32) c += __popc(matches(u));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
  if (lane == 0) s_wc[w] = c;
  __syncthreads();
  unsigned base = 0;
  for (int k = 0; k < w; ++k) base += s_wc[k];
  if (base < n && base + s_wc[w] >= n) {  // this warp holds the n-th: walk its units in order
    unsigned run = base;
    for (int64_t u0 = a; u0 < b; u0 += 32) {
      const int64_t u = u0 + lane;
      const unsigned bits = u < b ? matches(u) : 0u;
      unsigned incl = __popc(bits);
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
      }
      const unsigned before = run + incl - __popc(bits);
      if (before < n && run + incl >= n) {  // in this lane's unit: the (n - before)-th set bit
        unsigned need = n - before, bb = bits;
        for (int e = 0; e < E; ++e) {
          if (bb & 1u) {
            if (--need == 0) {
              *s_v = u * E + e;
              break;
            }
          }
          bb >>= 1;
        }
      }
      run += __shfl_sync(0xffffffffu, incl, 31);
      if (run >= n) break;
    }
  }
  __syncthreads();
  return *s_v;
}

// Order key of a bf16 logit from its 16 bits (order_key of the widened
// value, shifted down 16), the value of a key, and the widened value's
// 32-bit order key (its low half is fixed by the sign).
__device__ __forceinline__ uint32_t order_key16(uint32_t h) {
  h &= 0xFFFFu;
  if (h == 0x8000u) h = 0u;
  return (h & 0x8000u) ? (~h & 0xFFFFu) : (h | 0x8000u);
}
__device__ __forceinline__ float key16_value(uint32_t key) {
  const uint32_t h = (key & 0x8000u) ? (key & 0x7FFFu) : (~key & 0xFFFFu);
  return __uint_as_float(h << 16);
}
__device__ __forceinline__ uint32_t key16_to_key32(uint32_t key) {
  return (key << 16) | ((key & 0x8000u) ? 0u : 0xFFFFu);
}

// bf16 counters are indexed by bit pattern: pattern h in half h & 1 of word
// h >> 1. In key order (descending value), key word kw (keys 2kw+1, 2kw)
// lives in pattern word kw - 16384 for kw >= 16384 (non-negative values, the
// higher key in the high half) and in pattern word 32767 - kw below (negative
// values, the higher key in the low half).
__device__ __forceinline__ int pattern_word(int kw) { return kw >= 16384 ? kw - 16384 : 32767 - kw; }

// Count the tokens of every bit pattern of a bf16 row (-0 as +0); the thread
// that loads token `tok` (-1: none) returns its pattern in *tokbits.
template <bool VEC>
__device__ __forceinline__ void count_patterns(const char* row, int64_t V, uint32_t* cnt, int tok, uint32_t* tokbits) {
  if constexpr (VEC) {
    constexpr int U = 4;
    const int Vu = static_cast<int>(V / 8);
    for (int u0 = threadIdx.x; u0 < Vu; u0 += U * kNucThreads) {
      uint4 w[U];
#pragma unroll
      for (int h = 0; h < U; ++h) {
        const int u = u0 + h * kNucThreads;
        w[h] = u < Vu ? ldg16(reinterpret_cast<const uint4*>(row) + u) : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int h = 0; h < U; ++h) {
        const int u = u0 + h * kNucThreads;
        if (u >= Vu) break;
        uint32_t ws[4] = {w[h].x, w[h].y, w[h].z, w[h].w};
        if ((tok >> 3) == u) *tokbits = (ws[(tok & 7) >> 1] >> (16 * (tok & 1))) & 0xFFFFu;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint32_t x = ws[c] ^ (__vcmpeq2(ws[c], 0x80008000u) & 0x80008000u);  // -0 -> +0
          atomicAdd(&cnt[(x >> 1) & 0x7FFFu], 1u << ((x & 1u) << 4));
          atomicAdd(&cnt[x >> 17], 1u << (((x >> 16) & 1u) << 4));
        }
      }
    }
  } else {
    const unsigned short* r16 = reinterpret_cast<const unsigned short*>(row);
    for (int64_t v = threadIdx.x; v < V; v += kNucThreads) {
      uint32_t x = __ldg(r16 + v);
      if (v == tok) *tokbits = x;
      if (x == 0x8000u) x = 0u;
      atomicAdd(&cnt[x >> 1], 1u << ((x & 1u) << 4));
    }
  }
}

// Counts of the two keys of key word kw, the higher key first.
__device__ __forceinline__ void kword_counts(const uint32_t* cnt, int kw, uint32_t (&c)[2]) {
  const uint32_t wv = cnt[pattern_word(kw)];
  const uint32_t lo = wv & 0xFFFFu, hi = wv >> 16;
  c[0] = kw >= 16384 ? hi : lo;
  c[1] = kw >= 16384 ? lo : hi;
}

// ... and their fixed-point masses count * round(2^((x - m) k) 2^kFix).
__device__ __forceinline__ void kword_mass(const uint32_t* cnt, int kw, float m, float k, uint32_t (&c)[2],
                                           unsigned long long (&mass)[2]) {
  kword_counts(cnt, kw, c);
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    mass[t] = 0ull;
    if (c[t]) {
      const uint32_t key = 2u * static_cast<uint32_t>(kw) + 1u - t;
      mass[t] = static_cast<unsigned long long>(c[t]) * to_fixed(ex2((key16_value(key) - m) * k));
    }
  }
}

// fp32 rows, and bf16 rows whose counters wrapped: the row maximum, whether
// the row holds a NaN, and the drafted token's logit (the thread that loads
// it). Called by the whole block; the results are in shared memory.
template <int DT, bool VEC>
__device__ __forceinline__ void max_pass(const char* row, int64_t V, int tok, float* s_wmax, int* s_bad, float* s_xg,
                                         float& m, bool& bad) {
  constexpr int E = VEC ? Elem<DT>::kPerVec : 1;
  const int64_t Vu = V / E;
  float mx = -INFINITY;
  bool nan = false;
  for (int64_t u = threadIdx.x; u < Vu; u += kNucThreads) {
    float x[E];
    if constexpr (VEC) Elem<DT>::unpack(ldg16(reinterpret_cast<const uint4*>(row) + u), x);
    else x[0] = Elem<DT>::at(row, u);
#pragma unroll
    for (int e = 0; e < E; ++e) {
      nan |= x[e] != x[e];
      mx = fmaxf(mx, x[e]);
      if (u * E + e == tok) *s_xg = x[e];
    }
  }
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  nan = __any_sync(0xffffffffu, nan);
  if (lane == 0) s_wmax[w] = mx;
  if (nan && lane == 0) *s_bad = 1;
  __syncthreads();
  m = -INFINITY;
  for (int q = 0; q < kNucWarps; ++q) m = fmaxf(m, s_wmax[q]);
  bad = *s_bad != 0 || !isfinite(m);
  __syncthreads();
}

// Radix descent (fp32 rows, and bf16 rows whose counters could have
// overflowed): the cut key kappa, the mass above it, the row's whole mass and
// the target; also the tokens at the cut value (c) and the mass of each
// (each). Called by the whole block; `hist` is 4096 64-bit bins.
template <int DT, bool VEC>
__device__ __forceinline__ void radix_cut(const char* row, int64_t V, float m, float k, double top_p,
                                          unsigned long long* hist, unsigned* s_cnt, unsigned long long* s_tmp,
                                          int* s_d, unsigned long long* s_above, unsigned long long& whole,
                                          unsigned long long& target, unsigned long long& above, uint32_t& kappa,
                                          unsigned& c, unsigned long long& each) {
  const int tid = threadIdx.x;
  constexpr bool bf16 = DT == 1;
  for (int i = tid; i < kNucBins; i += kNucThreads) hist[i] = 0ull;
  for (int i = tid; i < kNucCountBins; i += kNucThreads) s_cnt[i] = 0u;
  __syncthreads();
  // digit 1: bits 31..20, every token; its total is the row's whole mass
  digit_pass<DT, VEC>(row, V, m, k, 0u, 0u, 20, 0xFFFu, false, hist, s_cnt);
  __syncthreads();
  unsigned long long local = 0;
  for (int i = tid; i < kNucBins; i += kNucThreads) local += hist[i];
  const unsigned long long excl = block_scan_u64(local, s_tmp);
  if (tid == kNucThreads - 1) *s_above = excl + local;
  __syncthreads();
  whole = *s_above;
  target = static_cast<unsigned long long>(ceil(top_p * static_cast<double>(whole)));
  if (target < 1ull) target = 1ull;
  if (target > whole) target = whole;
  __syncthreads();
  find_digit(hist, kNucBins, 0ull, target, s_tmp, s_d, s_above);
  uint32_t prefix = static_cast<uint32_t>(*s_d) << 20, pmask = 0xFFF00000u;
  above = *s_above;
  const int shift = bf16 ? 16 : 8;      // digit 2: bits 19..16 complete a widened bf16 key; fp32: 19..8
  const int nb = bf16 ? 16 : kNucBins;
  __syncthreads();
  for (int i = tid; i < kNucBins; i += kNucThreads) hist[i] = 0ull;
  __syncthreads();
  digit_pass<DT, VEC>(row, V, m, k, prefix, pmask, shift, static_cast<uint32_t>(nb - 1), bf16, hist, s_cnt);
  __syncthreads();
  find_digit(hist, nb, above, target, s_tmp, s_d, s_above);
  int dl = *s_d;
  prefix |= static_cast<uint32_t>(dl) << shift;
  above = *s_above;
  if (bf16) {
    kappa = prefix | ((prefix & 0x80000000u) ? 0u : 0xFFFFu);  // the low half of a widened bf16 key
  } else {  // digit 3: bits 7..0, with token counts
    __syncthreads();
    for (int i = tid; i < kNucCountBins; i += kNucThreads) hist[i] = 0ull;
    __syncthreads();
    digit_pass<DT, VEC>(row, V, m, k, prefix, 0xFFFFFF00u, 0, 0xFFu, true, hist, s_cnt);
    __syncthreads();
    find_digit(hist, kNucCountBins, above, target, s_tmp, s_d, s_above);
    dl = *s_d;
    above = *s_above;
    kappa = prefix | static_cast<uint32_t>(dl);
  }
  // (the crossing bin holds mass, hence at least one token; the guards only keep every division defined)
  c = s_cnt[dl];
  each = c ? hist[dl] / c : 1ull;  // every token of the cut value has the same mass
  __syncthreads();
}

template <int DT, bool VEC>
__global__ void __launch_bounds__(kNucThreads, 1) k_nucleus(NucleusArgs a) {
  // dynamic shared memory: a 128 KiB region (bf16 counters, or the radix
  // path's 4096 64-bit bins), then the walk (rowoff[B + 1], base[B])
  extern __shared__ unsigned long long nuc_smem[];
  uint32_t* cnt = reinterpret_cast<uint32_t*>(nuc_smem);
  unsigned long long* hist = nuc_smem;
  int* walk_smem = reinterpret_cast<int*>(nuc_smem + kValueWords / 2);
  __shared__ unsigned s_cnt[kNucCountBins];
  __shared__ unsigned long long s_tmp[kNucWarps + 1];
  __shared__ int s_itmp[kNucWarps + 1];
  __shared__ unsigned s_wc[kNucWarps];
  __shared__ unsigned long long s_step[kNucThreads];  // bf16: mass of each 32-word step, descending keys
  __shared__ unsigned s_wtok[kNucWarps];
  __shared__ int s_wkey[kNucWarps];
  __shared__ float s_wmax[kNucWarps];
  __shared__ int s_sel, s_bad, s_tok;
  __shared__ const char* s_row;
  __shared__ uint32_t s_tokbits;
  __shared__ float s_xg;
  __shared__ int s_d;
  __shared__ unsigned long long s_above, s_each;
  __shared__ unsigned s_c;
  __shared__ uint32_t s_kappa;
  __shared__ long long s_v;
  pdl_wait();
  pdl_trigger();
  const RowSpace& rs = a.rs;
  const Walk w{walk_smem, walk_smem + rs.B + 1};
  const int64_t nrows = build_walk<kNucThreads>(rs, walk_smem, s_itmp);
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  for (int64_t r = blockIdx.x; r < nrows; r += gridDim.x) {
    if (a.only && !__ldcg(a.only + r)) continue;  // the fast path served this row (block-uniform)
    if (tid == 0) {
      const int32_t* tokp;
      s_row = locate<DT>(rs, w, r, tokp);
      int tok = load_token(tokp);
      if (tok >= a.V) tok = -1;  // out of range: flagged by the sampling kernel, nothing to record
      s_tok = tok;
      s_bad = 0;
      s_tokbits = 0u;
      s_xg = 0.f;
    }
    __syncthreads();
    const char* row = s_row;
    const int tok = s_tok;
    float m = 0.f;
    bool bad = false;
    unsigned long long whole = 0, target = 0, above = 0, each = 1;
    unsigned c = 0;
    uint32_t kappa = 0;
    bool radix = DT == 0;
    if constexpr (DT == 1) {
      for (int i = tid; i < kValueWords / 4; i += kNucThreads) reinterpret_cast<uint4*>(cnt)[i] = make_uint4(0, 0, 0, 0);
      __syncthreads();
      count_patterns<VEC>(row, a.V, cnt, tok, &s_tokbits);
      __syncthreads();
      // the largest value present, and whether a NaN or +inf is present (patterns 0x7F80.. and 0xFF81..)
      int kmax = -1;
      unsigned ntok = 0;
      for (int st = 0; st < 32; ++st) {
        const int kw = kValueWords - 1 - 32 * (32 * wid + st) - lane;  // descending key words
        uint32_t cc[2];
        kword_counts(cnt, kw, cc);
        ntok += cc[0] + cc[1];
        if (cc[1]) kmax = max(kmax, 2 * kw);
        if (cc[0]) kmax = max(kmax, 2 * kw + 1);
        const int rw = pattern_word(kw);  // patterns 2rw, 2rw+1
        const uint32_t p0 = 2u * rw, wv = cnt[rw];
        const bool nonfin = ((wv & 0xFFFFu) && ((p0 & 0x7FFFu) >= 0x7F80u) && p0 != 0xFF80u) ||
                            ((wv >> 16) && (((p0 + 1u) & 0x7FFFu) >= 0x7F80u));
        if (nonfin) s_bad = 1;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
        ntok += __shfl_xor_sync(0xffffffffu, ntok, o);
      }
      if (lane == 0) {
        s_wkey[wid] = kmax;
        s_wtok[wid] = ntok;
      }
      __syncthreads();
      int kmx = -1;
      unsigned tokens = 0;
      for (int q = 0; q < kNucWarps; ++q) {
        kmx = max(kmx, s_wkey[q]);
        tokens += s_wtok[q];
      }
      m = kmx >= 0 ? key16_value(static_cast<uint32_t>(kmx)) : NAN;
      bad = s_bad != 0 || !isfinite(m);
      if (tid == 0) s_xg = __uint_as_float(s_tokbits << 16);
      if (tokens != static_cast<unsigned>(a.V)) {
        radix = true;  // a value with more than 65,535 tokens wrapped its counter
      } else if (!bad) {
        // step t = 32 wid + st covers key words 32767 - 32 t down to 32767 - 32 t - 31, one per lane: the
        // mass of every step, a block scan over the 1024 steps, then the one step that holds the crossing
        for (int st = 0; st < 32; ++st) {
          const int t = 32 * wid + st;
          uint32_t cc[2];
          unsigned long long mm[2];
          kword_mass(cnt, kValueWords - 1 - 32 * t - lane, m, a.k, cc, mm);
          unsigned long long sm = mm[0] + mm[1];
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) sm += __shfl_xor_sync(0xffffffffu, sm, o);
          if (lane == 0) s_step[t] = sm;
        }
        if (tid == 0) {
          s_c = 0u;
          s_sel = 0;
        }
        __syncthreads();
        const unsigned long long mine = s_step[tid];
        const unsigned long long ex = block_scan_u64(mine, s_tmp);
        if (tid == kNucThreads - 1) s_above = ex + mine;  // the whole mass: the normaliser, scaled by 2^42
        __syncthreads();
        whole = s_above;
        target = static_cast<unsigned long long>(ceil(a.top_p * static_cast<double>(whole)));
        if (target < 1ull) target = 1ull;
        if (target > whole) target = whole;
        __syncthreads();  // every thread has read the whole mass from s_above
        if (ex < target && ex + mine >= target) {  // this step holds the crossing
          s_sel = tid;
          s_above = ex;
        }
        __syncthreads();
        if (wid == 0) {  // walk the one step: a warp scan over its 32 key words
          const int kw = kValueWords - 1 - 32 * s_sel - lane;
          uint32_t cc[2];
          unsigned long long mm[2];
          kword_mass(cnt, kw, m, a.k, cc, mm);
          const unsigned long long lm = mm[0] + mm[1];
          unsigned long long incl = lm;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const unsigned long long t = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += t;
          }
          const unsigned long long xa = s_above + incl - lm;  // mass of every larger value
          __syncwarp();
          if (xa < target && xa + mm[0] >= target) {  // the higher key of the word
            s_kappa = 2u * static_cast<uint32_t>(kw) + 1u;
            s_above = xa;
            s_c = cc[0];
            s_each = mm[0] / cc[0];
          } else if (xa + mm[0] < target && xa + lm >= target) {
            s_kappa = 2u * static_cast<uint32_t>(kw);
            s_above = xa + mm[0];
            s_c = cc[1];
            s_each = mm[1] / cc[1];
          }
        }
        __syncthreads();
        kappa = key16_to_key32(s_kappa);
        above = s_above;
        c = s_c;
        each = s_each ? s_each : 1ull;
      }
      __syncthreads();
    }
    if (radix) {
      max_pass<DT, VEC>(row, a.V, tok, s_wmax, &s_bad, &s_xg, m, bad);
      if (!bad)
        radix_cut<DT, VEC>(row, a.V, m, a.k, a.top_p, hist, s_cnt, s_tmp, &s_d, &s_above, whole, target, above,
                           kappa, c, each);
    }
    if (bad) {  // a non-finite row: the sampling kernel flags the request
      if (tid == 0) {
        a.row_m[r] = NAN;
        a.row_lf[r] = NAN;
        a.cut_key[r] = 0u;
        a.cut_v[r] = static_cast<int32_t>(a.V - 1);
        if (tok >= 0) rs.xg[r] = s_xg;
      }
      __syncthreads();
      continue;
    }
    // tokens at the cut value: how many are needed, and which is the last
    const unsigned long long need = (target - above + each - 1) / each;
    const unsigned take = static_cast<unsigned>(need < c ? need : c);
    const unsigned long long kept = above + static_cast<unsigned long long>(take) * each;
    int64_t vcut = a.V - 1;
    if (take > 0 && take < c) vcut = nth_equal<DT, VEC>(row, a.V, kappa, take, s_wc, &s_v);
    if (tid == 0) {
      a.row_m[r] = m;
      a.row_lf[r] = log(static_cast<double>(kept)) - kFix * 0.6931471805599453;
      a.cut_key[r] = kappa;
      a.cut_v[r] = static_cast<int32_t>(vcut);
      if (tok >= 0) rs.xg[r] = s_xg;
    }
    __syncthreads();
  }
}

// ---------------------------------------------------------------- fast path
//
// k_nucleus_fast, bf16 rows of 16-byte vectors: the cut is found inside a
// narrow window of values chosen from a sample, so a token costs one
// exponential and a few compares, and only the tokens inside the window are
// counted; a row the window does not serve is handed to k_nucleus (flag 1).
//  1. sample: 512 evenly spaced 16-byte units (4,096 logits); their maximum
//     is the row's reference r (masses are 2^((x - r) k), relative to r);
//  2. a histogram of the sample's masses over 4,096 bins of 16 consecutive
//     16-bit order keys; scanning it from the top brackets the crossing of
//     top_p: the bins between mass fractions top_p - delta and top_p + delta,
//     delta four standard errors of the sample's estimate (effective size
//     (sum q)^2 / sum q^2) plus 0.002, form the window, at most 1,024 keys
//     (narrowed around the estimated crossing when wider), never reaching the
//     patterns of infinities and NaNs;
//  3. one HBM pass: every token adds its mass to the total (fp32 per 16-byte
//     unit, fp64 per thread), tokens above the window also to the mass above,
//     and tokens inside it are counted per value (shared reductions);
//  4. the window's values, from the top, each with mass count * 2^((x - r) k)
//     (exact in fp64): the value where the mass above plus the running sum
//     reaches top_p * total is the cut. When the crossing lies above (below)
//     the window, one more pass counts the 1,024 keys just above (below) it;
//     when it misses again, or the row holds a NaN or an infinity, the row is
//     flagged;
//  5. the tie cut, as in k_nucleus.
// Rows are never wrong for a poor sample, only handed over: every mass that
// decides the cut is summed over the whole row.
constexpr int kFastThreads = 256;
constexpr int kFastWarps = kFastThreads / 32;
constexpr int kSampleUnits = 2 * kFastThreads;
constexpr int kSampleBins = 4096;  // 16 keys each
constexpr int kWinKeys = 1024;
constexpr int kFiniteKeyLo = 0x0080, kFiniteKeyHi = 0xFF7F;  // keys of -max finite and +max finite

__device__ __forceinline__ unsigned long long pack_f2(float lo, float hi) {
  unsigned long long v;
  asm("mov.b64 %0, {%1, %2};" : "=l"(v) : "f"(lo), "f"(hi));
  return v;
}
__device__ __forceinline__ void unpack_f2(unsigned long long v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ unsigned long long add_f2(unsigned long long a, unsigned long long b) {
  unsigned long long d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ unsigned long long mul_f2(unsigned long long a, unsigned long long b) {
  unsigned long long d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ void red_if(uint32_t addr, uint32_t v, uint32_t limit) {  // count at addr when v <= limit
  asm volatile("{\n\t.reg .pred p;\n\tsetp.le.u32 p, %1, %2;\n\t@p red.shared.add.u32 [%0], 1;\n\t}"
               :: "r"(addr), "r"(v), "r"(limit) : "memory");
}

// One warp's share [ua, ub) (16-byte units) of a bf16 row for k_nucleus_fast:
// the row's mass 2^((x - r) k) summed (fp32 per unit, two tokens at a time in
// packed f32x2 arithmetic, fp64 across units), the part of it above the key
// window [klo, khi], and a count per window key in this warp's counters
// (shared address wcnt). The window index of a token comes from its bf16
// bits h, by the window's place:
//   MODE 1, window below zero (khi <= 0x7FFE): key = 0xFFFF - h for every
//     negative value; every non-negative value (-0 too) lies above;
//   MODE 2, window above zero (klo >= 0x8001): key = h + 0x8000 for every
//     positive value; h sign-extended puts every negative pattern and both
//     zeros below;
//   MODE 0, any window: the 32-bit order key of x + 0 (so -0 counts as +0),
//     f ^ ((f >> 31) | 0x80000000), whose top half is the 16-bit key.
// A NaN lands above or below the window and its mass poisons the total.
template <int MODE>
__device__ __forceinline__ void window_unit(const uint4& v, unsigned long long nrr2, unsigned long long kk2, int klo,
                                            int khi, uint32_t wcnt, double& tot, double& above) {
  const int span = khi - klo;
  const int c1 = 0xFFFF - klo, c2 = 0x8000 - klo;
  const uint32_t klo32 = static_cast<uint32_t>(klo) << 16, khi32 = (static_cast<uint32_t>(khi) << 16) | 0xFFFFu;
  const uint32_t ws[4] = {v.x, v.y, v.z, v.w};
  unsigned long long ts2 = 0ull;
  float as = 0.f;
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const uint32_t f[2] = {ws[c] << 16, ws[c] & 0xFFFF0000u};
    float e[2], q[2];
    unpack_f2(mul_f2(add_f2(pack_f2(__uint_as_float(f[0]), __uint_as_float(f[1])), nrr2), kk2), e[0], e[1]);
    q[0] = ex2(e[0]);
    q[1] = ex2(e[1]);
    ts2 = add_f2(ts2, pack_f2(q[0], q[1]));
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      if constexpr (MODE == 0) {
        const uint32_t g = __float_as_uint(__uint_as_float(f[half]) + 0.f);
        const uint32_t key32 = g ^ (static_cast<uint32_t>(static_cast<int32_t>(g) >> 31) | 0x80000000u);
        if (key32 > khi32) as += q[half];
        const uint32_t off = key32 - klo32;
        red_if(wcnt + ((off >> 16) << 2), off, khi32 - klo32);
      } else {
        const int idx = MODE == 1 ? c1 - static_cast<int>(f[half] >> 16) : (static_cast<int32_t>(f[half]) >> 16) + c2;
        if (idx > span) as += q[half];
        red_if(wcnt + (static_cast<uint32_t>(idx) << 2), static_cast<uint32_t>(idx), static_cast<uint32_t>(span));
      }
    }
  }
  float t0, t1;
  unpack_f2(ts2, t0, t1);
  tot += static_cast<double>(t0 + t1);
  above += static_cast<double>(as);
}

template <int MODE>
__device__ __forceinline__ void window_stream(const char* row, int ua, int ub, int lane, float rr, float kk, int klo,
                                              int khi, uint32_t wcnt, double& tot, double& above) {
  const unsigned long long nrr2 = pack_f2(-rr, -rr), kk2 = pack_f2(kk, kk);
  const uint4* src = reinterpret_cast<const uint4*>(row);
  constexpr int U = 4;
  int u0 = ua + lane;
  for (; u0 + 32 * (U - 1) < ub; u0 += 32 * U) {  // whole groups: no bounds checks
    uint4 wv[U];
#pragma unroll
    for (int h = 0; h < U; ++h) wv[h] = ldg16(src + u0 + 32 * h);
#pragma unroll
    for (int h = 0; h < U; ++h) window_unit<MODE>(wv[h], nrr2, kk2, klo, khi, wcnt, tot, above);
  }
  for (; u0 < ub; u0 += 32) window_unit<MODE>(ldg16(src + u0), nrr2, kk2, klo, khi, wcnt, tot, above);
}

__global__ void __launch_bounds__(kFastThreads, 4) k_nucleus_fast(NucleusArgs a) {
  extern __shared__ int walk_smem[];  // rowoff[B + 1], base[B]
  // one 32 KB area: the sample's bins (fp32), then the window's counters (one set per warp)
  __shared__ __align__(16) uint32_t s_area[kFastWarps * kWinKeys];
  float* const s_bm = reinterpret_cast<float*>(s_area);
  __shared__ float s_ftmp[kFastWarps + 1];
  __shared__ double s_dtmp[kFastWarps + 1];
  __shared__ double s_red[2 * kFastWarps];
  __shared__ float s_fred[2 * kFastWarps];
  __shared__ int s_itmp[kFastWarps + 1];
  __shared__ unsigned s_wc[kFastWarps];
  __shared__ const char* s_row;
  __shared__ int s_tok, s_bhi, s_blo, s_bst, s_klo, s_khi, s_kappa, s_wsel;
  __shared__ float s_xg;
  __shared__ double s_before, s_qk;
  __shared__ unsigned s_ck, s_nth;
  __shared__ long long s_v;
  pdl_wait();
  pdl_trigger();
  const RowSpace& rs = a.rs;
  const Walk w{walk_smem, walk_smem + rs.B + 1};
  const int64_t nrows = build_walk<kFastThreads>(rs, walk_smem, s_itmp);
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int Vu = static_cast<int>(a.V / 8);
  const float kk = a.k;
  for (int64_t r = blockIdx.x; r < nrows; r += gridDim.x) {
    if (tid == 0) {
      const int32_t* tokp;
      s_row = locate<1>(rs, w, r, tokp);
      int tok = load_token(tokp);
      if (tok >= a.V) tok = -1;
      s_tok = tok;
      s_xg = tok >= 0 ? __uint_as_float(static_cast<uint32_t>(__ldg(reinterpret_cast<const unsigned short*>(s_row) + tok)) << 16)
                      : 0.f;
      s_bhi = s_blo = s_bst = -1;
    }
    for (int i = tid; i < kSampleBins; i += kFastThreads) s_bm[i] = 0.f;
    __syncthreads();
    const char* row = s_row;
    const int tok = s_tok;
    // 1. the sample (two units per thread, in registers) and its maximum
    float xs[16];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int j = tid + h * kFastThreads;
      const int u = static_cast<int>(((2ll * j + 1) * Vu) / (2 * kSampleUnits));
      float x8[8];
      Elem<1>::unpack(ldg16(reinterpret_cast<const uint4*>(row) + u), x8);
#pragma unroll
      for (int e = 0; e < 8; ++e) xs[8 * h + e] = x8[e];
    }
    float lm = -INFINITY;
#pragma unroll
    for (int e = 0; e < 16; ++e) lm = fmaxf(lm, xs[e]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) lm = fmaxf(lm, __shfl_xor_sync(0xffffffffu, lm, o));
    if (lane == 0) s_fred[wid] = lm;
    __syncthreads();
    float rr = -INFINITY;
    for (int q = 0; q < kFastWarps; ++q) rr = fmaxf(rr, s_fred[q]);
    const bool rok = isfinite(rr);
    // 2. the sample's masses over the bins
    float sq = 0.f, sq2 = 0.f;
    if (rok) {
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const float q = ex2((xs[e] - rr) * kk);
        if (q == q) {
          atomicAdd(&s_bm[order_key16(__float_as_uint(xs[e]) >> 16) >> 4], q);
          sq += q;
          sq2 += q * q;
        }
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      sq += __shfl_xor_sync(0xffffffffu, sq, o);
      sq2 += __shfl_xor_sync(0xffffffffu, sq2, o);
    }
    __syncthreads();  // every thread has read the maxima from s_fred
    if (lane == 0) {
      s_fred[wid] = sq;
      s_fred[kFastWarps + wid] = sq2;
    }
    __syncthreads();
    float stot = 0.f, stot2 = 0.f;
    for (int q = 0; q < kFastWarps; ++q) {
      stot += s_fred[q];
      stot2 += s_fred[kFastWarps + q];
    }
    const float tp = static_cast<float>(a.top_p);
    const float neff = stot2 > 0.f ? stot * stot / stot2 : 1.f;
    const float delta = 4.f * sqrtf(tp * (1.f - tp) / fmaxf(neff, 1.f)) + 0.002f;
    const float lo_t = (tp - delta) * stot, hi_t = (tp + delta) * stot, st_t = tp * stot;
    {  // thread t: bins 4095 - 16t down to 4080 - 16t; the first bins (from the top) past each threshold
      float c[16], sum = 0.f;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        c[j] = s_bm[kSampleBins - 1 - 16 * tid - j];
        sum += c[j];
      }
      float run = block_scan<float, kFastThreads>(sum, s_ftmp);
      int bhi = -1, blo = -1, bst = -1;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        run += c[j];
        const int b = kSampleBins - 1 - 16 * tid - j;
        if (run > lo_t && bhi < 0) bhi = b;
        if (run >= hi_t && blo < 0) blo = b;
        if (run >= st_t && bst < 0) bst = b;
      }
      if (bhi >= 0) atomicMax(&s_bhi, bhi);
      if (blo >= 0) atomicMax(&s_blo, blo);
      if (bst >= 0) atomicMax(&s_bst, bst);
    }
    __syncthreads();
    if (tid == 0) {
      int bhi = s_bhi, blo = s_blo;
      if (blo < 0) blo = 0;  // top_p + delta is past the sample's mass: down to the lowest finite key
      if (bhi - blo + 1 > kWinKeys / 16) {  // too wide: around the estimated crossing
        bhi = min(bhi, s_bst + kWinKeys / 32 - 1);
        blo = max(blo, bhi - kWinKeys / 16 + 1);
      }
      const int klo = max(16 * blo, kFiniteKeyLo), khi = min(16 * bhi + 15, kFiniteKeyHi);
      s_klo = klo;
      s_khi = (!rok || bhi < 0 || khi < klo) ? -1 : khi;  // -1: no usable window
    }
    __syncthreads();
    if (s_khi < 0) {  // the exact kernel takes the row
      if (tid == 0) a.flags[r] = 1;
      __syncthreads();
      continue;
    }
    // 3./4. up to two passes; every decision below is block-uniform. Warp w streams units [w cw, (w+1) cw)
    //    and counts its window keys in its own counters, so the tie search reads one chunk again, not the
    //    row
    const int cw = (Vu + kFastWarps - 1) / kFastWarps;
    const int ua = min(Vu, wid * cw), ub = min(Vu, ua + cw);
    const uint32_t wcnt = static_cast<uint32_t>(__cvta_generic_to_shared(s_area + wid * kWinKeys));
    bool done = false, hand = false;
    double target = 0.0;
    for (int pass = 0; pass < 2 && !done && !hand; ++pass) {
      const int klo = s_klo, khi = s_khi;
      __syncthreads();  // every thread has read the window and, in the first pass, the sample's bins
      for (int i = tid; i < kFastWarps * kWinKeys; i += kFastThreads) s_area[i] = 0u;
      if (tid == 0) s_kappa = -1;
      __syncthreads();
      double tot = 0.0, above = 0.0;
      if (khi <= 0x7FFE) {
        window_stream<1>(row, ua, ub, lane, rr, kk, klo, khi, wcnt, tot, above);
      } else if (klo >= 0x8001) {
        window_stream<2>(row, ua, ub, lane, rr, kk, klo, khi, wcnt, tot, above);
      } else {
        window_stream<0>(row, ua, ub, lane, rr, kk, klo, khi, wcnt, tot, above);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        tot += __shfl_xor_sync(0xffffffffu, tot, o);
        above += __shfl_xor_sync(0xffffffffu, above, o);
      }
      if (lane == 0) {
        s_red[wid] = tot;
        s_red[kFastWarps + wid] = above;
      }
      __syncthreads();
      tot = 0.0;
      above = 0.0;
      for (int q = 0; q < kFastWarps; ++q) {
        tot += s_red[q];
        above += s_red[kFastWarps + q];
      }
      target = a.top_p * tot;
      const bool fin = isfinite(tot);
      // the window's values from the top (thread t: keys khi - 4t ... khi - 4t - 3)
      constexpr int KT = kWinKeys / kFastThreads;
      double wm = 0.0;
      float qk[KT];
      unsigned ck[KT];
#pragma unroll
      for (int t = 0; t < KT; ++t) ck[t] = 0u;
      const int top = khi - KT * tid;  // this thread's keys: top, top - 1, ..., top - KT + 1
#pragma unroll
      for (int t = 0; t < KT; ++t) {
        const int key = top - t;
        if (key >= klo) {
          const int idx = key - klo;
          unsigned sum = 0u;
#pragma unroll
          for (int v = 0; v < kFastWarps; ++v) sum += s_area[v * kWinKeys + idx];
          ck[t] = sum;
        }
        qk[t] = ck[t] ? ex2((key16_value(static_cast<uint32_t>(key)) - rr) * kk) : 0.f;
        wm += static_cast<double>(ck[t]) * static_cast<double>(qk[t]);
      }
      const double ex = block_scan<double, kFastThreads>(wm, s_dtmp);
      if (fin && above < target) {
        double run = above + ex;
#pragma unroll
        for (int t = 0; t < KT; ++t) {
          const double mass = static_cast<double>(ck[t]) * static_cast<double>(qk[t]);
          if (ck[t] && run < target && run + mass >= target) {
            s_kappa = top - t;
            s_before = run;
            s_qk = static_cast<double>(qk[t]);
            s_ck = ck[t];
          }
          run += mass;
        }
      }
      __syncthreads();
      if (!fin) {
        hand = true;
      } else if (s_kappa >= 0) {
        done = true;
      } else if (pass == 0) {  // the crossing lies above (below) the window: count the keys just above (below)
        const bool up = !(above < target);
        if (up ? khi >= kFiniteKeyHi : klo <= kFiniteKeyLo) {
          hand = true;
        } else if (tid == 0) {  // read by every thread after the barrier that opens the next pass
          if (up) {
            s_klo = khi + 1;
            s_khi = min(khi + kWinKeys, kFiniteKeyHi);
          } else {
            s_khi = klo - 1;
            s_klo = max(klo - kWinKeys, kFiniteKeyLo);
          }
        }
      } else {
        hand = true;
      }
      if (!done && !hand) __syncthreads();  // s_klo / s_khi written
    }
    // the reference r must lie close enough to the row's maximum that exp(-lf) stays a normal float for the
    // sampling kernel
    if (!done || s_before + static_cast<double>(s_ck) * s_qk > 1e26) {
      if (tid == 0) a.flags[r] = 1;
      __syncthreads();
      continue;
    }
    const uint32_t kappa = key16_to_key32(static_cast<uint32_t>(s_kappa));
    const double before = s_before, q = s_qk;
    const unsigned c = s_ck;
    double need = ceil((target - before) / q);
    if (need < 1.0) need = 1.0;
    const unsigned take = need < static_cast<double>(c) ? static_cast<unsigned>(need) : c;
    const double kept = before + static_cast<double>(take) * q;
    int64_t vcut = a.V - 1;
    if (take < c) {  // the chunk that holds the take-th token at the cut value, then that token within it
      if (tid == 0) {
        const int idx = s_kappa - s_klo;
        unsigned n = take;
        int sel = kFastWarps - 1;
        for (int v = 0; v < kFastWarps; ++v) {
          const unsigned cv = s_area[v * kWinKeys + idx];
          if (n <= cv) {
            sel = v;
            break;
          }
          n -= cv;
        }
        s_wsel = sel;
        s_nth = n;
      }
      __syncthreads();
      const int sa = min(Vu, s_wsel * cw), sb = min(Vu, sa + cw);
      vcut = 8ll * sa + nth_equal<1, true, kFastWarps>(row + 16ll * sa, 8ll * (sb - sa), kappa, s_nth, s_wc, &s_v);
    }
    if (tid == 0) {
      a.flags[r] = 0;
      a.row_m[r] = rr;  // the reference of the masses: lf is relative to it
      a.row_lf[r] = log(kept);
      a.cut_key[r] = kappa;
      a.cut_v[r] = static_cast<int32_t>(vcut);
      if (tok >= 0) rs.xg[r] = s_xg;
    }
    __syncthreads();
  }
}

cudaError_t launch_nucleus_fast(const NucleusArgs& a, cudaStream_t st) {
  const size_t smem = static_cast<size_t>(2 * a.rs.B + 1) * sizeof(int);
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t rows_max = static_cast<int64_t>(a.rs.B) * ((a.rs.K + 1) * a.rs.L + 1);
  const dim3 grid(static_cast<unsigned>(std::max<int64_t>(1, std::min<int64_t>(rows_max, 4 * sms))));
  if (smem > 48 * 1024) {
    const cudaError_t e =
        cudaFuncSetAttribute(k_nucleus_fast, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  return launch_pdl(k_nucleus_fast, grid, dim3(kFastThreads), smem, st, a);
}

cudaError_t launch_nucleus(const NucleusArgs& a, int dtype, bool vec, cudaStream_t st) {
  const size_t smem = kValueWords * sizeof(uint32_t) + static_cast<size_t>(2 * a.rs.B + 1) * sizeof(int);
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t rows_max = static_cast<int64_t>(a.rs.B) * ((a.rs.K + 1) * a.rs.L + 1);
  const dim3 grid(static_cast<unsigned>(std::max<int64_t>(1, std::min<int64_t>(rows_max, sms))));
  auto go = [&](auto kernel) {
    const cudaError_t e =
        cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    return launch_pdl(kernel, grid, dim3(kNucThreads), smem, st, a);
  };
  if (dtype == 0) return vec ? go(k_nucleus<0, true>) : go(k_nucleus<0, false>);
  return vec ? go(k_nucleus<1, true>) : go(k_nucleus<1, false>);
}

}  // namespace specv
