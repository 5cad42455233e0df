// The per-request accept decision, shared by both verify paths.
//
// Speculative sampling with rejection correction ("DBLAST: Dependent Block
// Drafting for Stochastic Speculative Decoding", Pith review, "Assumptions"):
// position i is accepted iff u_i < min(1, p_i(x_i) / q_i(x_i)); the verifier
// stops at the first rejection. For a latent-mixture draft ("What carries the
// argument", Eq. 5) q_i is the mixture marginal under the category posterior
// pi_i(z) ∝ q(z|y) prod_{k<i} q_k(x_k|y,z).
#pragma once

#include "common.cuh"

namespace specv {

constexpr int kMaxL = 32;
constexpr int kMaxK = 8;
constexpr int kMaxRows = (kMaxK + 1) * kMaxL;

// Inputs of one request's decision, in shared memory. Row q of the request:
// q < ell is target position q; q = ell + z*ell + i is draft (z, i).
struct DecideIn {
  const float* xg;   // raw logit at the drafted token, per row
  const float* m;    // row max of raw logits
  const float* s;    // sum 2^((x - m) log2e / T)
  const double* ls;  // log(s) in fp64, per row (read when K > 1)
  const double* lw;  // log q(z|y) in fp64 [K], nullptr for w = 1 (K == 1)
  const int* x;      // drafted tokens [ell]
  int ell, K, L;
  float T;
};

// Terminal-row parameters: p(v) = 2^((x_t - mt) k) * ct, q(v) = sum_z 2^((x_z - mz) k) * cz.
struct DecideOut {
  int j;
  int bad;            // a non-finite posterior or ratio at or before j
  float ct, mt;
  float cz[kMaxK], mz[kMaxK];
};

// Run by the 32 lanes of one warp (lane i tests position i). A fast pass
// computes every ratio rho_i: for independent drafts in fp32 from the raw
// logit differences; with a posterior, the per-position log-probabilities
// and their prefix sums in fp64 (from fp64 log-normalisers) and only the
// K-way log-sum-exps and the final exponential in fp32. Its error in rho is
// below 1e-6 relative; only when some tested lane lies within 1e-5 of its
// threshold |u_i - min(1, rho_i)| or meets a non-finite value does the warp
// redo the decisions fully in fp64, where the normalisers are the only fp32
// quantities. u: this request's uniforms.
__device__ __forceinline__ DecideOut decide_warp_fp64(const DecideIn& in, const float* u);

__device__ __forceinline__ DecideOut decide_warp(const DecideIn& in, const float* u) {
  const int lane = threadIdx.x & 31;
  const int ell = in.ell, K = in.K;
  const bool act = lane < ell;
  const float invT = 1.f / in.T;
  const float uu = act ? u[lane] : 0.f;
  float rho = 1.f, lpi[kMaxK];
  bool finite = true;
#pragma unroll
  for (int z = 0; z < kMaxK; ++z) lpi[z] = 0.f;
  if (K == 1) {
    // rho = exp(((x_t - m_t) - (x_d - m_d)) / T + log(s_d / s_t))
    if (act) {
      const int q = ell + lane;
      const float d = ((in.xg[lane] - in.m[lane]) - (in.xg[q] - in.m[q])) * invT + logf(in.s[q] / in.s[lane]);
      rho = expf(d);
      finite = isfinite(d) && isfinite(in.xg[q]) && isfinite(in.xg[lane]);
    }
  } else {
    const double invTd = 1.0 / static_cast<double>(in.T);
    double lqz[kMaxK], lpd[kMaxK], amax = -INFINITY;
#pragma unroll
    for (int z = 0; z < kMaxK; ++z) {
      lqz[z] = 0.0;
      lpd[z] = 0.0;
      if (z < K) {
        if (act) {
          const int q = ell + z * ell + lane;
          lqz[z] = static_cast<double>(in.xg[q] - in.m[q]) * invTd - in.ls[q];  // x - m is exact in fp32
        }
        double v = __shfl_up_sync(0xffffffffu, lqz[z], 1);
        if (lane == 0) v = 0.0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const double t = __shfl_up_sync(0xffffffffu, v, o);
          if (lane >= o) v += t;
        }
        lpd[z] = (in.lw ? in.lw[z] : 0.0) + v;
        amax = fmax(amax, lpd[z]);
      }
    }
    float sa = 0.f;
#pragma unroll
    for (int z = 0; z < kMaxK; ++z)
      if (z < K) sa += expf(static_cast<float>(lpd[z] - amax));
    const double norm = amax + static_cast<double>(logf(sa));
    double tmax = -INFINITY;
#pragma unroll
    for (int z = 0; z < kMaxK; ++z) {
      if (z < K) {
        lpd[z] -= norm;
        lpi[z] = static_cast<float>(lpd[z]);
        tmax = fmax(tmax, lpd[z] + lqz[z]);
      }
    }
    float st = 0.f;
#pragma unroll
    for (int z = 0; z < kMaxK; ++z)
      if (z < K) st += expf(static_cast<float>(lpd[z] + lqz[z] - tmax));
    const double lq = tmax + static_cast<double>(logf(st));
    const double lp = act ? static_cast<double>(in.xg[lane] - in.m[lane]) * invTd - in.ls[lane] : 0.0;
    rho = expf(static_cast<float>(lp - lq));
    finite = isfinite(norm) && isfinite(lp) && isfinite(lq);
  }
  const float thr = fminf(1.f, rho);
  constexpr float band = 1e-5f;
  const bool close = act && (!finite || isnan(rho) || fabsf(uu - thr) < band);
  if (__any_sync(0xffffffffu, close)) return decide_warp_fp64(in, u);
  const unsigned stop = __ballot_sync(0xffffffffu, act && !(uu < thr));
  DecideOut o;
  o.j = stop ? __ffs(stop) - 1 : ell;
  o.bad = 0;
  o.ct = o.mt = 0.f;
  const int src = o.j & 31;
  float lpj[kMaxK];
#pragma unroll
  for (int z = 0; z < kMaxK; ++z) lpj[z] = __shfl_sync(0xffffffffu, lpi[z], src);
  if (o.j < ell) {
    o.ct = 1.f / in.s[o.j];
    o.mt = in.m[o.j];
#pragma unroll
    for (int z = 0; z < kMaxK; ++z) {
      if (z < K) {
        const int q = ell + z * ell + o.j;
        o.cz[z] = expf(lpj[z]) / in.s[q];
        o.mz[z] = in.m[q];
      } else {
        o.cz[z] = 0.f;
        o.mz[z] = 0.f;
      }
    }
  }
  return o;
}

__device__ __forceinline__ DecideOut decide_warp_fp64(const DecideIn& in, const float* u) {
  const int lane = threadIdx.x & 31;
  const int ell = in.ell, K = in.K;
  const double T = static_cast<double>(in.T);
  const bool act = lane < ell;
  double lp = 0.0, lqz[kMaxK];
#pragma unroll
  for (int z = 0; z < kMaxK; ++z) lqz[z] = 0.0;
  if (act) {
    lp = (static_cast<double>(in.xg[lane]) - static_cast<double>(in.m[lane])) / T -
         log(static_cast<double>(in.s[lane]));
#pragma unroll
    for (int z = 0; z < kMaxK; ++z) {
      if (z < K) {
        const int q = ell + z * ell + lane;
        lqz[z] = (static_cast<double>(in.xg[q]) - static_cast<double>(in.m[q])) / T -
                 log(static_cast<double>(in.s[q]));
      }
    }
  }
  // log pi_i(z) = log w_z + sum_{k<i} log q_k(x_k|y,z) - logsumexp_z(.); for K = 1
  // this is exactly 0 and q_i = q_i(.|y), the independent proposal.
  double lpi[kMaxK];
  double amax = -INFINITY;
#pragma unroll
  for (int z = 0; z < kMaxK; ++z) {
    lpi[z] = 0.0;
    if (z < K) {
      double v = __shfl_up_sync(0xffffffffu, lqz[z], 1);
      if (lane == 0) v = 0.0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const double t = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += t;
      }
      const double lw = in.lw ? in.lw[z] : 0.0;
      lpi[z] = lw + v;
      amax = fmax(amax, lpi[z]);
    }
  }
  double sa = 0.0;
#pragma unroll
  for (int z = 0; z < kMaxK; ++z)
    if (z < K) sa += exp(lpi[z] - amax);
  const double norm = amax + log(sa);
  double tmax = -INFINITY;
#pragma unroll
  for (int z = 0; z < kMaxK; ++z) {
    if (z < K) {
      lpi[z] -= norm;
      tmax = fmax(tmax, lpi[z] + lqz[z]);
    }
  }
  double st = 0.0;
#pragma unroll
  for (int z = 0; z < kMaxK; ++z)
    if (z < K) st += exp(lpi[z] + lqz[z] - tmax);
  const double lq = tmax + log(st);
  const double rho = exp(lp - lq);
  const bool bad = !isfinite(norm) || isnan(rho);
  const double thr = fmin(1.0, rho);
  const float uu = act ? u[lane] : 0.f;
  const bool acc = static_cast<double>(uu) < thr;
  const unsigned stop = __ballot_sync(0xffffffffu, act && (bad || !acc));
  DecideOut o;
  o.j = stop ? __ffs(stop) - 1 : ell;
  o.bad = (__shfl_sync(0xffffffffu, bad ? 1 : 0, o.j & 31) && stop) ? 1 : 0;
  o.ct = o.mt = 0.f;
  // terminal multipliers, from lane j (residual draw)
  const int src = o.j & 31;
  double lpj[kMaxK];
#pragma unroll
  for (int z = 0; z < kMaxK; ++z) lpj[z] = __shfl_sync(0xffffffffu, z < K ? lpi[z] : 0.0, src);
  if (o.j < ell) {
    o.ct = static_cast<float>(1.0 / static_cast<double>(in.s[o.j]));
    o.mt = in.m[o.j];
#pragma unroll
    for (int z = 0; z < kMaxK; ++z) {
      if (z < K) {
        const int q = ell + z * ell + o.j;
        o.cz[z] = static_cast<float>(exp(lpj[z]) / static_cast<double>(in.s[q]));
        o.mz[z] = in.m[q];
      } else {
        o.cz[z] = 0.f;
        o.mz[z] = 0.f;
      }
    }
  }
  return o;
}

// ------------------------------------------------- top-p filtered decisions

// Inputs of one request's decision when every row is filtered to its top-p
// nucleus ("DBLAST", Pith review, "What would settle it" and "Assumptions":
// target probabilities under the same sampling filter). Row layout as in
// DecideIn. The filtered log-probability of the drafted token in row q is
// (xg - m) / T - lf when the token is in the row's nucleus (in[q] != 0),
// else -inf; lf is the log of the row's nucleus mass sum 2^((x - m) k).
struct DecideTopP {
  const float* xg;
  const float* m;
  const double* lf;
  const unsigned char* in;
  const double* lw;  // log q(z|y) [K], nullptr for w = 1 (K == 1)
  int ell, K, L;
  float T;
};

// log sum exp over the first K entries; -inf when every entry is -inf.
__device__ __forceinline__ double lse_k(const double* a, int K) {
  double m = -INFINITY;
#pragma unroll
  for (int z = 0; z < kMaxK; ++z)
    if (z < K) m = fmax(m, a[z]);
  if (m == -INFINITY) return -INFINITY;
  double s = 0.0;
#pragma unroll
  for (int z = 0; z < kMaxK; ++z)
    if (z < K) s += exp(a[z] - m);
  return m + log(s);
}

// Run by the 32 lanes of one warp (lane i tests position i), in fp64 with
// the filtered rows. A token outside the target's nucleus has p = 0 and is
// rejected (rho = 0); a token the filtered proposal gives 0 has rho = +inf
// and is accepted; a posterior whose normaliser is not finite (every
// category gives an accepted token probability 0) marks the request bad.
__device__ __forceinline__ DecideOut decide_warp_topp(const DecideTopP& in, const float* u) {
  const int lane = threadIdx.x & 31;
  const int ell = in.ell, K = in.K;
  const double T = static_cast<double>(in.T);
  const bool act = lane < ell;
  double lp = 0.0, lqz[kMaxK];
#pragma unroll
  for (int z = 0; z < kMaxK; ++z) lqz[z] = 0.0;
  if (act) {
    lp = in.in[lane] ? (static_cast<double>(in.xg[lane]) - static_cast<double>(in.m[lane])) / T - in.lf[lane]
                     : -INFINITY;
#pragma unroll
    for (int z = 0; z < kMaxK; ++z) {
      if (z < K) {
        const int q = ell + z * ell + lane;
        lqz[z] = in.in[q] ? (static_cast<double>(in.xg[q]) - static_cast<double>(in.m[q])) / T - in.lf[q]
                          : -INFINITY;
      }
    }
  }
  // log pi_i(z) = log w_z + sum_{k<i} log q_k(x_k|y,z) - logsumexp_z(.)
  double lpi[kMaxK];
#pragma unroll
  for (int z = 0; z < kMaxK; ++z) {
    lpi[z] = -INFINITY;
    if (z < K) {
      double v = __shfl_up_sync(0xffffffffu, lqz[z], 1);
      if (lane == 0) v = 0.0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const double t = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += t;
      }
      lpi[z] = (in.lw ? in.lw[z] : 0.0) + v;
    }
  }
  const double norm = lse_k(lpi, K);
  const bool bad = !isfinite(norm);
  double t[kMaxK];
#pragma unroll
  for (int z = 0; z < kMaxK; ++z) {
    lpi[z] = bad ? -INFINITY : lpi[z] - norm;
    t[z] = lpi[z] + lqz[z];
  }
  const double lq = lse_k(t, K);
  const double rho = lp == -INFINITY ? 0.0 : exp(lp - lq);
  const double thr = fmin(1.0, rho);
  const float uu = act ? u[lane] : 0.f;
  const bool acc = static_cast<double>(uu) < thr;
  const unsigned stop = __ballot_sync(0xffffffffu, act && (bad || isnan(rho) || !acc));
  DecideOut o;
  o.j = stop ? __ffs(stop) - 1 : ell;
  o.bad = (__shfl_sync(0xffffffffu, (bad || isnan(rho)) ? 1 : 0, o.j & 31) && stop) ? 1 : 0;
  o.ct = o.mt = 0.f;
  const int src = o.j & 31;
  double lpj[kMaxK];
#pragma unroll
  for (int z = 0; z < kMaxK; ++z) lpj[z] = __shfl_sync(0xffffffffu, lpi[z], src);
  if (o.j < ell) {  // terminal multipliers of the residual at j: p = 2^((x - mt) k) ct, q = sum_z 2^((x - mz) k) cz
    o.ct = static_cast<float>(exp(-in.lf[o.j]));
    o.mt = in.m[o.j];
#pragma unroll
    for (int z = 0; z < kMaxK; ++z) {
      if (z < K) {
        const int q = ell + z * ell + o.j;
        o.cz[z] = static_cast<float>(exp(lpj[z] - in.lf[q]));
        o.mz[z] = in.m[q];
      } else {
        o.cz[z] = 0.f;
        o.mz[z] = 0.f;
      }
    }
  }
  return o;
}

// ------------------------------------------------------------ terminal draw

struct Best {
  double score;
  int idx;
};

// Higher score wins; equal scores go to the lower token.
__device__ __forceinline__ void best_merge(Best& a, const Best& b) {
  if (b.score > a.score || (b.score == a.score && b.idx >= 0 && (a.idx < 0 || b.idx < a.idx))) a = b;
}

__device__ __forceinline__ void warp_best(Best& v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    Best w;
    w.score = __shfl_xor_sync(0xffffffffu, v.score, o);
    w.idx = __shfl_xor_sync(0xffffffffu, v.idx, o);
    best_merge(v, w);
  }
}

}  // namespace specv
