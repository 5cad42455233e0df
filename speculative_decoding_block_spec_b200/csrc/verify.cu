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
// Grid (P, B): the P blocks of request b each
//   1. read the request's verify length, drafted tokens and the logits at
//      those tokens (inputs only, before waiting on the statistics grid);
//   2. merge the statistics partials of the request's rows;
//   3. in warp 0, run the accept tests in fp64 (posterior by a warp scan over
//      positions) and find j with a ballot — identically in every block;
//   4. scan 1/P of row j (target, K draft rows, Gumbel row) for the best
//      residual and bonus scores;
// and the last block to finish (atomic ticket, reset by that block) merges
// the P partials and writes the outputs.
#include <algorithm>

#include "common.cuh"
#include "decide.cuh"
#include "internal.h"

namespace specv {

__device__ __forceinline__ void block_best(Best& v, Best* red) {
  warp_best(v);
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[w] = v;
  __syncthreads();
  if (w == 0) {
    v = lane < kWarps ? red[lane] : Best{-INFINITY, -1};
    warp_best(v);
  }
  __syncthreads();
}

template <int DT>
__device__ __forceinline__ const char* req_row(const VerifyArgs& a, int b, int64_t toff, int ell, int q) {
  constexpr int64_t esz = Elem<DT>::kBytes;
  if (q < ell) return static_cast<const char*>(a.target) + (toff + q) * a.V * esz;
  const int q2 = q - ell, z = q2 / ell, i = q2 - z * ell;
  return static_cast<const char*>(a.draft) + ((static_cast<int64_t>(b) * a.K + z) * a.L + i) * a.V * esz;
}

template <int DT, bool VEC>
__global__ void __launch_bounds__(kThreads) k_accept_sample(VerifyArgs a, float k) {
  __shared__ int s_x[kMaxL];
  __shared__ float s_xg[kMaxRows];  // raw logit at the drafted token, per request row
  __shared__ float s_m[kMaxRows], s_s[kMaxRows];
  __shared__ float s_c[kMaxK + 1], s_mm[kMaxK + 1];
  __shared__ int s_flags, s_j, s_last;
  __shared__ int s_cnt[2 * kWarps];
  __shared__ Best s_red[kWarps];

  const int b = blockIdx.y, p = blockIdx.x, tid = threadIdx.x, lane = tid & 31;
  const int L = a.L, K = a.K;
  const int64_t V = a.V;

  // ---- 1. inputs only
  int ell = a.vlen ? a.vlen[b] : L;
  const bool bad_len = ell < 0 || ell > L;
  if (bad_len) ell = 0;
  if (tid == 0) s_flags = bad_len ? kFlagVerifyLen : 0;
  __syncthreads();
  if (tid < ell) {
    int x = a.tokens[static_cast<int64_t>(b) * L + tid];
    if (x < 0 || x >= V) {
      atomicOr(&s_flags, kFlagTokenRange);
      x = 0;
    }
    s_x[tid] = x;
  }
  __syncthreads();
  const int64_t toff = a.row_off ? static_cast<int64_t>(a.row_off[b]) : static_cast<int64_t>(b) * (L + 1);
  const int nb = (K + 1) * ell;
  for (int q = tid; q < nb; q += kThreads) {
    const int i = q < ell ? q : (q - ell) % ell;
    s_xg[q] = Elem<DT>::at(req_row<DT>(a, b, toff, ell, q), s_x[i]);
  }

  pdl_wait();
  pdl_trigger();

  // ---- 2. statistics of this request's rows
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
  const int64_t rowbase = static_cast<int64_t>(before) * (K + 1);
  const int64_t N = static_cast<int64_t>(total) * (K + 1) * a.Vu;
  for (int q = tid; q < nb; q += kThreads) {
    const int64_t r = rowbase + q;
    const int64_t c0 = split_owner(r * a.Vu, N, a.G), c1 = split_owner((r + 1) * a.Vu - 1, N, a.G);
    float m = -INFINITY, s = 0.f;
    for (int64_t c = c0; c <= c1; ++c) {
      if (split_start(c + 1, N, a.G) == split_start(c, N, a.G)) continue;  // empty share: no partial
      const float2 pr = a.rpart[c + r];
      ms_merge(m, s, pr.x, pr.y, k);
    }
    s_m[q] = m;
    s_s[q] = s;
    if (!isfinite(m) || !isfinite(s)) atomicOr(&s_flags, kFlagNonFinite);
  }
  __syncthreads();

  // ---- 3. accept tests (fp64), first rejection by ballot
  if (tid < 32 && s_flags == 0) {
    const DecideIn in{s_xg, s_m, s_s, s_x, ell, K, L, a.T};
    const DecideOut o = decide_warp(in, a.u + static_cast<int64_t>(b) * L,
                                    a.mix_w ? a.mix_w + static_cast<int64_t>(b) * K : nullptr);
    if (lane == 0) {
      s_j = o.j;
      if (o.bad) s_flags |= kFlagNonFinite;
      s_c[0] = o.ct;
      s_mm[0] = o.mt;
      for (int z = 0; z < K; ++z) {
        s_c[1 + z] = o.cz[z];
        s_mm[1 + z] = o.mz[z];
      }
    }
  }
  __syncthreads();
  const int flags = s_flags;

  // ---- 4. this block's share of the terminal row
  Best br{-INFINITY, -1}, bb{-INFINITY, -1};
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
  }
  block_best(br, s_red);
  block_best(bb, s_red);
  if (tid == 0) a.tpart[static_cast<int64_t>(b) * a.P + p] = TermPart{br.score, bb.score, br.idx, bb.idx, {0, 0}};

  // ---- last block of the request: merge and write
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    s_last = atomicAdd(&a.tickets[b], 1) == a.P - 1;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  if (tid < 32) {
    Best r{-INFINITY, -1}, o{-INFINITY, -1};
    for (int c = lane; c < a.P; c += 32) {
      const TermPart* tp = a.tpart + static_cast<int64_t>(b) * a.P + c;
      best_merge(r, Best{__ldcg(&tp->res_score), __ldcg(&tp->res_idx)});
      best_merge(o, Best{__ldcg(&tp->bon_score), __ldcg(&tp->bon_idx)});
    }
    warp_best(r);
    warp_best(o);
    const int j = s_j;
    const int t = (flags == 0) ? ((j < ell && r.idx >= 0) ? r.idx : o.idx) : -1;
    const bool ok = flags == 0 && t >= 0;
    int32_t* out = a.out_tokens + static_cast<int64_t>(b) * (L + 1);
    for (int i = lane; i <= L; i += 32) out[i] = !ok ? -1 : (i < j ? s_x[i] : (i == j ? t : -1));
    if (lane == 0) {
      a.accept_len[b] = ok ? j : -1;
      if (flags) atomicOr(a.status, flags);
      else if (!ok) atomicOr(a.status, kFlagNonFinite);
      a.tickets[b] = 0;
    }
  }
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
