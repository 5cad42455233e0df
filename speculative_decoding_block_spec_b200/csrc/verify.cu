// Accept tests, first rejection and the terminal Gumbel-max draw.
//
// Speculative sampling with rejection correction ("DBLAST: Dependent Block
// Drafting for Stochastic Speculative Decoding", Pith review, "Assumptions",
// after Leviathan et al. and Chen et al.): position i is accepted iff
// u_i < min(1, p_i(x_i) / q_i(x_i)); the first rejection j ends the block and
// the last token is drawn from norm(max(0, p_j - q_j)); with no rejection a
// bonus token is drawn from target row l. For a latent-mixture draft ("What
// carries the argument", Eq. 5) q_i is the mixture marginal under the
// category posterior pi_i(z) ∝ q(z|y) prod_{k<i} q_k(x_k|y,z).
//
// Grid (P, B), launched after the statistics kernel with programmatic
// dependent launch. The P blocks of request b each
//   1. merge the statistics partials of the request's window rows and read the
//      drafted-token logits the statistics kernel recorded;
//   2. take the accept decisions in one warp (decide_warp) — identically in
//      every block, so no block waits for another;
//   3. score 1/P of terminal row j (target, K draft rows, Gumbel row) and
//      publish each warp's best residual and bonus candidates as 64-bit
//      order-preserving keys with red.max (no return, no wait).
// The last block of the grid to finish (atomic ticket) writes every
// request's accepted length and tokens and clears the keys, so the workspace
// is ready for the next call.
#include <algorithm>

#include "common.cuh"
#include "decide.cuh"
#include "internal.h"

namespace specv {

// Order-preserving 64-bit key of a terminal candidate: the fp64 score with its
// lowest 20 bits replaced by (2^20 - 1 - token), so that an unsigned max picks
// the highest score and, among scores equal to 32 significant bits, the lowest
// token. 0 means "no candidate". Needs V <= 2^20.
__device__ __forceinline__ unsigned long long score_key(double score, int idx) {
  if (idx < 0) return 0ull;
  unsigned long long bits = static_cast<unsigned long long>(__double_as_longlong(score));
  bits = (bits >> 63) ? ~bits : (bits | (1ull << 63));
  return (bits & ~0xFFFFFull) | (0xFFFFFull - static_cast<unsigned long long>(idx));
}
__device__ __forceinline__ int key_token(unsigned long long key) {
  return key ? static_cast<int>(0xFFFFFull - (key & 0xFFFFFull)) : -1;
}
__device__ __forceinline__ void red_max_u64(unsigned long long* p, unsigned long long v) {
  asm volatile("red.relaxed.gpu.global.max.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

// Owner block of unit e in the even split, without a 64-bit integer division.
__device__ __forceinline__ int64_t owner_of(int64_t e, int64_t N, int64_t G) {
  const int64_t num = (e + 1) * G - 1;
  int64_t q = static_cast<int64_t>(static_cast<double>(num) / static_cast<double>(N));
  while (q > 0 && q * N > num) --q;
  while ((q + 1) * N <= num) ++q;
  return q;
}

template <int DT, bool VEC>
__global__ void __launch_bounds__(kThreads) k_accept_sample(VerifyArgs a, float k) {
  __shared__ float s_xg[kMaxRows];  // logit at the drafted token, per request row
  __shared__ float s_m[kMaxRows], s_s[kMaxRows];
  __shared__ int s_x[kMaxL];
  __shared__ float s_c[kMaxK + 1], s_mm[kMaxK + 1];
  __shared__ int s_flags, s_j, s_last;
  __shared__ int s_cnt[2 * kWarps];

  const int b = blockIdx.y, p = blockIdx.x, tid = threadIdx.x, lane = tid & 31;
  const int L = a.L, K = a.K;
  const int64_t V = a.V;

  int ell = a.vlen ? a.vlen[b] : L;
  const bool bad_len = ell < 0 || ell > L;
  if (bad_len) ell = 0;
  if (tid == 0) s_flags = bad_len ? kFlagVerifyLen : 0;
  const int64_t toff = a.row_off ? static_cast<int64_t>(a.row_off[b]) : static_cast<int64_t>(b) * (L + 1);

  pdl_wait();
  pdl_trigger();

  // ---- 1. this request's rows: offset in the statistics walk, partials, token logits
  int before = 0, total = 0;
  for (int bb = tid; bb < a.B; bb += kThreads) {
    int l = a.vlen ? a.vlen[bb] : L;
    if (l < 0 || l > L) l = 0;
    total += l;
    if (bb < b) before += l;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    before += __shfl_xor_sync(0xffffffffu, before, o);
    total += __shfl_xor_sync(0xffffffffu, total, o);
  }
  if (lane == 0) {
    s_cnt[tid >> 5] = before;
    s_cnt[kWarps + (tid >> 5)] = total;
  }
  __syncthreads();
  before = 0;
  total = 0;
  for (int w = 0; w < kWarps; ++w) {
    before += s_cnt[w];
    total += s_cnt[kWarps + w];
  }
  const int nb = (K + 1) * ell;
  const int64_t rowbase = static_cast<int64_t>(before) * (K + 1);
  const int64_t N = static_cast<int64_t>(total) * (K + 1) * a.Vu;
  if (tid < ell) {
    const int x = a.tokens[static_cast<int64_t>(b) * L + tid];
    if (x < 0 || x >= V) atomicOr(&s_flags, kFlagTokenRange);
    s_x[tid] = x;
  }
  for (int q = tid; q < nb; q += kThreads) {
    const int64_t r = rowbase + q;
    const int64_t c0 = owner_of(r * a.Vu, N, a.G), c1 = owner_of((r + 1) * a.Vu - 1, N, a.G);
    const float xq = __ldcg(a.xg + r);
    float m = -INFINITY, s = 0.f;
    for (int64_t c = c0; c <= c1; c += 4) {  // 4 independent loads in flight per round trip
      float2 pr[4];
#pragma unroll
      for (int t = 0; t < 4; ++t)  // blocks with an empty share (only when N < grid) wrote nothing
        pr[t] = c + t <= c1 && (N >= a.G || split_start(c + t + 1, N, a.G) > split_start(c + t, N, a.G))
                    ? __ldcg(a.rpart + c + t + r)
                    : make_float2(-INFINITY, 0.f);
#pragma unroll
      for (int t = 0; t < 4; ++t) ms_merge(m, s, pr[t].x, pr[t].y, k);
    }
    s_m[q] = m;
    s_s[q] = s;
    s_xg[q] = xq;
    if (!isfinite(m) || !isfinite(s)) atomicOr(&s_flags, kFlagNonFinite);
  }
  __syncthreads();

  // ---- 2. accept tests, first rejection by ballot
  if (tid < 32) {
    int j = ell;
    if (s_flags == 0) {
      const DecideIn in{s_xg, s_m, s_s, s_x, ell, K, L, a.T};
      const DecideOut o = decide_warp(in, a.u + static_cast<int64_t>(b) * L,
                                      a.mix_w ? a.mix_w + static_cast<int64_t>(b) * K : nullptr);
      j = o.j;
      if (lane == 0) {
        if (o.bad) s_flags |= kFlagNonFinite;
        s_c[0] = o.ct;
        s_mm[0] = o.mt;
        for (int z = 0; z < K; ++z) {
          s_c[1 + z] = o.cz[z];
          s_mm[1 + z] = o.mz[z];
        }
      }
    }
    if (lane == 0) {
      s_j = j;
      if (p == 0) {  // for the block that writes the outputs
        a.dec[b].j = j;
        a.dec[b].flags = s_flags;
      }
    }
  }
  __syncthreads();
  const int flags = s_flags;

  // ---- 3. this block's share of the terminal row; each warp publishes its maxima
  if (flags == 0) {
    const int j = s_j;
    const bool resid = j < ell;
    const double invT = 1.0 / static_cast<double>(a.T);
    const char* trow = static_cast<const char*>(a.target) + (toff + j) * V * Elem<DT>::kBytes;
    const float* grow = a.g + (static_cast<int64_t>(b) * (L + 1) + j) * V;
    const float mt = resid ? s_mm[0] : 0.f, ct = resid ? s_c[0] : 0.f;
    constexpr int E = VEC ? Elem<DT>::kPerVec : 1;
    const int64_t Vu = V / E;
    const int64_t u1 = (static_cast<int64_t>(p) + 1) * Vu / a.P;
    Best br{-INFINITY, -1}, bb{-INFINITY, -1};
    for (int64_t u = static_cast<int64_t>(p) * Vu / a.P + tid; u < u1; u += kThreads) {
      float xt[E], gv[E], q[E];
      if constexpr (VEC) {
        Elem<DT>::unpack(ldg16(reinterpret_cast<const uint4*>(trow) + u), xt);
#pragma unroll
        for (int h = 0; h < E / 4; ++h) {
          const uint4 w = ldg16(reinterpret_cast<const uint4*>(grow + u * E) + h);
          gv[4 * h] = __uint_as_float(w.x); gv[4 * h + 1] = __uint_as_float(w.y);
          gv[4 * h + 2] = __uint_as_float(w.z); gv[4 * h + 3] = __uint_as_float(w.w);
        }
      } else {
        xt[0] = Elem<DT>::at(trow, u);
        gv[0] = __ldg(grow + u);
      }
#pragma unroll
      for (int e = 0; e < E; ++e) {
        const Best c{static_cast<double>(xt[e]) * invT + static_cast<double>(gv[e]), static_cast<int>(u * E + e)};
        if (c.score > bb.score) bb = c;
        q[e] = 0.f;
      }
      if (resid) {
        for (int z = 0; z < K; ++z) {
          const char* drow =
              static_cast<const char*>(a.draft) + ((static_cast<int64_t>(b) * K + z) * L + j) * V * Elem<DT>::kBytes;
          float xd[E];
          if constexpr (VEC) Elem<DT>::unpack(ldg16(reinterpret_cast<const uint4*>(drow) + u), xd);
          else xd[0] = Elem<DT>::at(drow, u);
          const float cz = s_c[1 + z], mz = s_mm[1 + z];
#pragma unroll
          for (int e = 0; e < E; ++e) q[e] = fmaf(cz, ex2((xd[e] - mz) * k), q[e]);
        }
#pragma unroll
        for (int e = 0; e < E; ++e) {
          const float r = ex2((xt[e] - mt) * k) * ct - q[e];
          if (r > 0.f) {
            const Best c{static_cast<double>(lg2(r) * kLn2) + static_cast<double>(gv[e]), static_cast<int>(u * E + e)};
            if (c.score > br.score) br = c;
          }
        }
      }
    }
    warp_best(br);
    warp_best(bb);
    if (lane == 0) {
      if (br.idx >= 0) red_max_u64(a.keys + 2 * b, score_key(br.score, br.idx));
      if (bb.idx >= 0) red_max_u64(a.keys + 2 * b + 1, score_key(bb.score, bb.idx));
    }
  }

  // ---- the last block of the grid writes every request's outputs
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = atomicAdd(a.tickets, 1) == static_cast<int>(gridDim.x * gridDim.y) - 1;
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  for (int t = tid; t < a.B * (L + 1); t += kThreads) {
    const int rb = t / (L + 1), i = t - rb * (L + 1);
    int l = a.vlen ? a.vlen[rb] : L;
    if (l < 0 || l > L) l = 0;
    const int j = __ldcg(&a.dec[rb].j), f = __ldcg(&a.dec[rb].flags);
    const unsigned long long kr = __ldcg(a.keys + 2 * rb), kb = __ldcg(a.keys + 2 * rb + 1);
    const int tk = i < j ? __ldg(a.tokens + static_cast<int64_t>(rb) * L + i) : -1;
    const int term = f ? -1 : ((j < l && kr) ? key_token(kr) : key_token(kb));
    const bool ok = f == 0 && term >= 0;
    a.out_tokens[static_cast<int64_t>(rb) * (L + 1) + i] = !ok ? -1 : (i < j ? tk : (i == j ? term : -1));
    if (i == 0) {
      a.accept_len[rb] = ok ? j : -1;
      if (f) atomicOr(a.status, f);
      else if (!ok) atomicOr(a.status, kFlagNonFinite);
    }
  }
  __syncthreads();  // every output thread has read the keys before they are cleared
  for (int t = tid; t < 2 * a.B; t += kThreads) a.keys[t] = 0ull;
  if (tid == 0) *a.tickets = 0;
}

cudaError_t launch_accept_sample(const VerifyArgs& a, int dtype, bool vec, cudaStream_t st) {
  const float k = static_cast<float>(1.4426950408889634 / static_cast<double>(a.T));
  const dim3 grid(a.P, a.B), block(kThreads);
  if (dtype == 0)
    return vec ? launch_pdl(k_accept_sample<0, true>, grid, block, 0, st, a, k)
               : launch_pdl(k_accept_sample<0, false>, grid, block, 0, st, a, k);
  return vec ? launch_pdl(k_accept_sample<1, true>, grid, block, 0, st, a, k)
             : launch_pdl(k_accept_sample<1, false>, grid, block, 0, st, a, k);
}

}  // namespace specv
