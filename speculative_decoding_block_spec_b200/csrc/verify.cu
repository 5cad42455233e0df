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
//   0. read the request's tokens, uniforms and mixture weights while the
//      statistics kernel is still finishing;
//   1. merge the statistics partials of the request's window rows and read the
//      drafted-token logits the statistics kernel recorded;
//   2. take the accept decisions in one warp (decide_warp), identically in
//      every block, so no block waits for another; block 0 then writes the
//      accepted length and every output token but the terminal one;
//   3. score 1/P of terminal row j and publish each warp's best candidate as
//      a 64-bit order-preserving key with red.max (no return, no wait): after
//      a rejection the residual log(p - q) + g from the target, K draft and
//      Gumbel rows; with none, the bonus x / T + g from the target and Gumbel
//      rows.
// The last of the request's blocks to finish (per-request atomic ticket)
// writes the terminal token and clears the request's keys and ticket, so the
// workspace is ready for the next call. If rounding left no element with
// p > q after a rejection (impossible in exact arithmetic), that block draws
// row j by the bonus rule itself.
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

__device__ __forceinline__ int ticket_acq_rel(int* p) {
  int old;
  asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], 1;" : "=r"(old) : "l"(p) : "memory");
  return old;
}

// Owner block of unit e in the even split, without a 64-bit integer division.
__device__ __forceinline__ int64_t owner_of(int64_t e, int64_t N, int64_t G) {
  const int64_t num = (e + 1) * G - 1;
  int64_t q = static_cast<int64_t>(static_cast<double>(num) / static_cast<double>(N));
  while (q > 0 && q * N > num) --q;
  while ((q + 1) * N <= num) ++q;
  return q;
}

// Top-p membership of token v with logit x in terminal row t (0: target,
// 1 + z: draft category z): kept iff its order key is above the row's cut
// key, or equal to it with v at most the cut token. Always true unfiltered.
template <bool TP>
__device__ __forceinline__ bool kept(const uint32_t* ck, const int* cv, int t, float x, int64_t v) {
  if constexpr (!TP) {
    return true;
  } else {
    const uint32_t kx = order_key(x);
    return kx > ck[t] || (kx == ck[t] && v <= cv[t]);
  }
}

// Residual scores of two tokens of terminal row j (v < 0: skipped), with the
// arithmetic of the streaming scan: q = sum_z c_z 2^((x_z - m_z) k) in order
// z = 0..K-1, r = p - q by one fused multiply-add, score = ln r + g, or -inf
// when r <= 0. All loads of both tokens are issued before any is used.
template <int DT, bool TP>
__device__ __forceinline__ void residual_score2(const char* trow, const float* grow, const char* dbase,
                                                int64_t dstride, int K, const float* c, const float* mm, float k,
                                                const uint32_t* ck, const int* cv, int v1, int v2, double& s1,
                                                double& s2) {
  const int a1 = max(v1, 0), a2 = max(v2, 0);  // in-range addresses; skipped tokens are ignored below
  const float xt1 = Elem<DT>::at(trow, a1), xt2 = Elem<DT>::at(trow, a2);
  const float g1 = __ldg(grow + a1), g2 = __ldg(grow + a2);
  float xd1[kMaxK], xd2[kMaxK];
#pragma unroll
  for (int z = 0; z < kMaxK; ++z)
    if (z < K) {
      xd1[z] = Elem<DT>::at(dbase + z * dstride, a1);
      xd2[z] = Elem<DT>::at(dbase + z * dstride, a2);
    }
  float q1 = 0.f, q2 = 0.f;
#pragma unroll
  for (int z = 0; z < kMaxK; ++z)
    if (z < K) {
      q1 = fmaf(c[1 + z], kept<TP>(ck, cv, 1 + z, xd1[z], a1) ? ex2((xd1[z] - mm[1 + z]) * k) : 0.f, q1);
      q2 = fmaf(c[1 + z], kept<TP>(ck, cv, 1 + z, xd2[z], a2) ? ex2((xd2[z] - mm[1 + z]) * k) : 0.f, q2);
    }
  const float r1 = fmaf(kept<TP>(ck, cv, 0, xt1, a1) ? ex2((xt1 - mm[0]) * k) : 0.f, c[0], -q1);
  const float r2 = fmaf(kept<TP>(ck, cv, 0, xt2, a2) ? ex2((xt2 - mm[0]) * k) : 0.f, c[0], -q2);
  s1 = v1 >= 0 && r1 > 0.f ? static_cast<double>(lg2(r1) * kLn2) + static_cast<double>(g1) : -INFINITY;
  s2 = v2 >= 0 && r2 > 0.f ? static_cast<double>(lg2(r2) * kLn2) + static_cast<double>(g2) : -INFINITY;
}

// Slack of the residual pruning test, in natural-log units: far above the
// rounding of the bound and of the exact score (below 1e-5), so no element
// that could win is pruned.
constexpr float kPruneSlack = 4e-3f;

// KB: draft categories loaded together per terminal unit (1 for independent
// drafts, which then take two units per thread per iteration; 4 otherwise).
// TP: rows filtered to their top-p nuclei (cuts from the nucleus kernel).
template <int DT, bool VEC, int KB, bool TP>
__global__ void __launch_bounds__(kThreads, 3) k_accept_sample(VerifyArgs a, float k) {
  __shared__ float s_xg[kMaxRows];  // logit at the drafted token, per request row
  __shared__ float s_m[kMaxRows], s_s[kMaxRows];
  __shared__ unsigned char s_in[TP ? kMaxRows : 1];      // top-p: drafted token in the row's nucleus
  __shared__ uint32_t s_key[TP ? kMaxRows + 1 : 1];      // top-p: cut keys (last entry: the bonus row)
  __shared__ int s_cvr[TP ? kMaxRows + 1 : 1];           // top-p: cut tokens
  __shared__ uint32_t s_tk[kMaxK + 1];                   // top-p: cuts of the terminal rows (0: target)
  __shared__ int s_tv[kMaxK + 1];
  __shared__ int s_bbad;                                 // top-p: the bonus row is not finite
  __shared__ int s_x[kMaxL];
  __shared__ float s_u[kMaxL];
  __shared__ double s_lw[kMaxK], s_ls[kMaxRows];
  __shared__ float s_c[kMaxK + 1], s_mm[kMaxK + 1];
  __shared__ int s_flags, s_j, s_last, s_fail, s_scan;
  __shared__ Best s_best[kWarps];
  __shared__ int s_cnt[2 * kWarps];

  const int b = blockIdx.y, p = blockIdx.x, tid = threadIdx.x, lane = tid & 31;
  const int L = a.L, K = a.K;
  const int64_t V = a.V;
  int32_t* out = a.out_tokens + static_cast<int64_t>(b) * (L + 1);

  // ---- 0. inputs that do not come from the statistics kernel: read while it
  //         finishes (this grid starts early through programmatic launch)
  int ell = a.vlen ? a.vlen[b] : L;
  const bool bad_len = ell < 0 || ell > L;
  if (bad_len) ell = 0;
  if (tid == 0) s_flags = bad_len ? kFlagVerifyLen : 0;
  const int64_t toff = a.row_off ? static_cast<int64_t>(a.row_off[b]) : static_cast<int64_t>(b) * (L + 1);
  int before = b * L, total = a.B * L;  // verified positions of earlier requests, of all requests
  if (a.vlen) {
    before = 0;
    total = 0;
    for (int bb = tid; bb < a.B; bb += kThreads) {
      int l = a.vlen[bb];
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
  }
  __syncthreads();
  if (a.vlen) {
    before = 0;
    total = 0;
    for (int w = 0; w < kWarps; ++w) {
      before += s_cnt[w];
      total += s_cnt[kWarps + w];
    }
  }
  if (tid < ell) {
    const int x = a.tokens[static_cast<int64_t>(b) * L + tid];
    if (x < 0 || x >= V) atomicOr(&s_flags, kFlagTokenRange);
    s_x[tid] = x;
    s_u[tid] = a.u[static_cast<int64_t>(b) * L + tid];
  }
  if (tid < K && a.mix_w) s_lw[tid] = log(static_cast<double>(a.mix_w[static_cast<int64_t>(b) * K + tid]));

  pdl_wait();
  pdl_trigger();

  // ---- 1. this request's rows: merge the statistics partials (one round trip
  //         for up to 8 partials per row) and read the drafted-token logits;
  //         filtered: the nucleus kernel's maxima, normalisers and cuts
  if constexpr (TP) {
    __syncthreads();  // the drafted tokens (s_x) come from other threads
    // walk rows of request b: target 0..ell-1, bonus row ell, drafts (z, i) at ell + 1 + z*ell + i;
    // in shared memory the drafts sit at ell + z*ell + i and the bonus row at index kMaxRows
    const int nbt = (K + 1) * ell + 1;
    const int64_t rowbase = static_cast<int64_t>(before) * (K + 1) + b;
    for (int q = tid; q < nbt; q += kThreads) {
      const int64_t r = rowbase + q;
      const float m = __ldcg(a.nuc_m + r);
      const double lf = __ldcg(a.nuc_lf + r);
      const uint32_t ck = __ldcg(a.nuc_key + r);
      const int cv = __ldcg(a.nuc_v + r);
      if (q == ell) {  // its finiteness matters only if the last token is drawn from it
        s_key[kMaxRows] = ck;
        s_cvr[kMaxRows] = cv;
        s_bbad = !isfinite(m) || !isfinite(lf);
        continue;
      }
      const int d = q < ell ? q : q - 1;
      const int i = q < ell ? q : (q - ell - 1) % ell;
      const float xq = __ldcg(a.xg + r);
      const uint32_t kx = order_key(xq);
      s_m[d] = m;
      s_ls[d] = lf;
      s_xg[d] = xq;
      s_key[d] = ck;
      s_cvr[d] = cv;
      s_in[d] = (kx > ck || (kx == ck && s_x[i] <= cv)) ? 1 : 0;
      if (!isfinite(m) || !isfinite(lf)) atomicOr(&s_flags, kFlagNonFinite);
    }
    __syncthreads();
  }
  const int nb = TP ? 0 : (K + 1) * ell;
  const int64_t rowbase = static_cast<int64_t>(before) * (K + 1);
  const int64_t N = static_cast<int64_t>(total) * (K + 1) * a.Vu;
  for (int q = tid; q < nb; q += kThreads) {
    const int64_t r = rowbase + q;
    const int64_t c0 = owner_of(r * a.Vu, N, a.G), c1 = owner_of((r + 1) * a.Vu - 1, N, a.G);
    const float xq = __ldcg(a.xg + r);
    float m = -INFINITY, s = 0.f;
    for (int64_t c = c0; c <= c1; c += 8) {
      float2 pr[8];
#pragma unroll
      for (int t = 0; t < 8; ++t)  // blocks with an empty share (only when N < grid) wrote nothing
        pr[t] = c + t <= c1 && (N >= a.G || split_start(c + t + 1, N, a.G) > split_start(c + t, N, a.G))
                    ? __ldcg(a.rpart + c + t + r)
                    : make_float2(-INFINITY, 0.f);
#pragma unroll
      for (int t = 0; t < 8; ++t) ms_merge(m, s, pr[t].x, pr[t].y, k);
    }
    s_m[q] = m;
    s_s[q] = s;
    s_xg[q] = xq;
    if (K > 1) s_ls[q] = log(static_cast<double>(s));
    if (!isfinite(m) || !isfinite(s)) atomicOr(&s_flags, kFlagNonFinite);
  }
  __syncthreads();

  // ---- 2. accept tests and first rejection (warp 0, identically in every
  //         block); block 0 then writes every output but the terminal token
  if (tid < 32) {
    int j = ell, f = s_flags;
    if (f == 0) {
      DecideOut o;
      if constexpr (TP) {
        const DecideTopP in{s_xg, s_m, s_ls, s_in, a.mix_w ? s_lw : nullptr, ell, K, L, a.T};
        o = decide_warp_topp(in, s_u);
        if (o.j == ell && s_bbad) o.bad = 1;  // the bonus row is drawn from but is not finite
        if (lane <= K) {  // cuts of the terminal rows: target row j (or the bonus row), draft rows (z, j)
          const int jj = o.j;
          const int d = lane == 0 ? (jj < ell ? jj : kMaxRows) : ell + (lane - 1) * ell + jj;
          s_tk[lane] = lane == 0 || jj < ell ? s_key[d] : 0u;
          s_tv[lane] = lane == 0 || jj < ell ? s_cvr[d] : 0;
        }
      } else {
        const DecideIn in{s_xg, s_m, s_s, s_ls, a.mix_w ? s_lw : nullptr, s_x, ell, K, L, a.T};
        o = decide_warp(in, s_u);
      }
      j = o.j;
      if (o.bad) f |= kFlagNonFinite;
      if (lane == 0) {
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
      s_flags = f;
    }
    if (p == 0) {
      for (int i = lane; i <= L; i += 32)
        if (f || i != j) out[i] = (f == 0 && i < j) ? s_x[i] : -1;
      if (lane == 0) {
        a.accept_len[b] = f ? -1 : j;
        if (f) atomicOr(a.status, f);
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
    const char* dbase =
        static_cast<const char*>(a.draft) + (static_cast<int64_t>(b) * K * L + j) * V * Elem<DT>::kBytes;
    const int64_t dstride = static_cast<int64_t>(L) * V * Elem<DT>::kBytes;  // between draft categories
    const int64_t ua = static_cast<int64_t>(p) * Vu / a.P + tid;  // this thread's first unit
    bool stream = true;  // the full streaming scan below (every residual with the mixture drafts: its fallback)
    if constexpr (KB > 1) {
      if (resid) {
        // Mixture drafts: r = p - q <= p, so ln r(v) + g(v) <= ln p(v) + g(v) = bound(v), which needs only
        // the target and Gumbel rows: bound = ((x k + c1) ln 2) + g with c1 = log2(ct) - mt k. By the
        // Gumbel-max property about 1 / (residual mass) tokens of the row have a bound above the best
        // score, so the K draft rows are read only at a few tokens.
        // Pass 1: each thread keeps its two largest bounds (tokens w1, w2) and the third largest, t3,
        // which bounds every other token of its share.
        const float c1 = lg2(ct) - mt * k;
        float t1 = -INFINITY, t2 = -INFINITY, t3 = -INFINITY;
        int w1 = -1, w2 = -1;
        for (int64_t u0 = ua; u0 < u1; u0 += 2 * kThreads) {
          uint4 tv[2], gw[2][VEC ? E / 4 : 1];
          float xs[2], gs[2];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int64_t u = u0 + h * kThreads;
            if (u >= u1) break;
            if constexpr (VEC) {
              tv[h] = ldg16(reinterpret_cast<const uint4*>(trow) + u);
#pragma unroll
              for (int c = 0; c < E / 4; ++c) gw[h][c] = ldg16(reinterpret_cast<const uint4*>(grow + u * E) + c);
            } else {
              xs[h] = Elem<DT>::at(trow, u);
              gs[h] = __ldg(grow + u);
            }
          }
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int64_t u = u0 + h * kThreads;
            if (u >= u1) break;
            float xt[E], gv[E];
            if constexpr (VEC) {
              Elem<DT>::unpack(tv[h], xt);
#pragma unroll
              for (int c = 0; c < E / 4; ++c) {
                gv[4 * c] = __uint_as_float(gw[h][c].x); gv[4 * c + 1] = __uint_as_float(gw[h][c].y);
                gv[4 * c + 2] = __uint_as_float(gw[h][c].z); gv[4 * c + 3] = __uint_as_float(gw[h][c].w);
              }
            } else {
              xt[0] = xs[h];
              gv[0] = gs[h];
            }
#pragma unroll
            for (int e = 0; e < E; ++e) {
              const int v = static_cast<int>(u * E + e);
              const float bnd = kept<TP>(s_tk, s_tv, 0, xt[e], v) ? fmaf(fmaf(xt[e], k, c1), kLn2, gv[e]) : -INFINITY;
              if (bnd > t3) {
                if (bnd > t2) {
                  t3 = t2;
                  if (bnd > t1) {
                    t2 = t1; w2 = w1; t1 = bnd; w1 = v;
                  } else {
                    t2 = bnd; w2 = v;
                  }
                } else {
                  t3 = bnd;
                }
              }
            }
          }
        }
        // Round 1: the exact score of each warp's largest bound (8 tokens per block); their best is a
        // lower bound lb on the block's maximum. If none of them has p > q, round 1b scores every
        // thread's two candidates.
        bool ev1 = false, ev2 = false;  // w1 / w2 of this thread already scored
        float wt = t1;
        int wl = lane;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          const float ot = __shfl_xor_sync(0xffffffffu, wt, o);
          const int ol = __shfl_xor_sync(0xffffffffu, wl, o);
          if (ot > wt || (ot == wt && ol < wl)) {
            wt = ot;
            wl = ol;
          }
        }
        if (lane == wl && w1 >= 0) {
          double e1, unused;
          residual_score2<DT, TP>(trow, grow, dbase, dstride, K, s_c, s_mm, k, s_tk, s_tv, w1, -1, e1, unused);
          if (e1 > -INFINITY) best_merge(br, Best{e1, w1});
          ev1 = true;
        }
        double lb = -INFINITY;
        for (int round = 0; round < 2; ++round) {
          Best wb = br;
          warp_best(wb);
          if (lane == 0) s_best[tid >> 5] = wb;
          __syncthreads();
#pragma unroll
          for (int w = 0; w < kWarps; ++w) lb = fmax(lb, s_best[w].score);
          __syncthreads();
          if (lb > -INFINITY || round == 1) break;  // block-uniform
          double e1, e2;  // round 1b
          residual_score2<DT, TP>(trow, grow, dbase, dstride, K, s_c, s_mm, k, s_tk, s_tv, ev1 ? -1 : w1, w2, e1, e2);
          if (e1 > -INFINITY) best_merge(br, Best{e1, w1});
          if (e2 > -INFINITY) best_merge(br, Best{e2, w2});
          ev1 = ev2 = true;
        }
        if (lb > -INFINITY) {  // block-uniform
          stream = false;
          // Round 2: every token whose bound reaches lb - slack is scored exactly: this thread's w1 and
          // w2 if not yet scored, and, when its third bound reaches the cut too, every other token of
          // its share (read again, from L2).
          const float cut = static_cast<float>(lb) - kPruneSlack;
          const int q1 = (!ev1 && t1 >= cut) ? w1 : -1, q2 = (!ev2 && t2 >= cut) ? w2 : -1;
          if (q1 >= 0 || q2 >= 0) {
            double e1, e2;
            residual_score2<DT, TP>(trow, grow, dbase, dstride, K, s_c, s_mm, k, s_tk, s_tv, q1, q2, e1, e2);
            if (e1 > -INFINITY) best_merge(br, Best{e1, q1});
            if (e2 > -INFINITY) best_merge(br, Best{e2, q2});
          }
          if (t3 >= cut) {
            for (int64_t u = ua; u < u1; u += kThreads) {
              float xt[E], gv[E];
              if constexpr (VEC) {
                Elem<DT>::unpack(ldg16(reinterpret_cast<const uint4*>(trow) + u), xt);
#pragma unroll
                for (int c = 0; c < E / 4; ++c) {
                  const uint4 gq = ldg16(reinterpret_cast<const uint4*>(grow + u * E) + c);
                  gv[4 * c] = __uint_as_float(gq.x); gv[4 * c + 1] = __uint_as_float(gq.y);
                  gv[4 * c + 2] = __uint_as_float(gq.z); gv[4 * c + 3] = __uint_as_float(gq.w);
                }
              } else {
                xt[0] = Elem<DT>::at(trow, u);
                gv[0] = __ldg(grow + u);
              }
#pragma unroll
              for (int e = 0; e < E; ++e) {
                const int v = static_cast<int>(u * E + e);
                if (kept<TP>(s_tk, s_tv, 0, xt[e], v) && fmaf(fmaf(xt[e], k, c1), kLn2, gv[e]) >= cut && v != w1 &&
                    v != w2) {
                  double sc, unused;
                  residual_score2<DT, TP>(trow, grow, dbase, dstride, K, s_c, s_mm, k, s_tk, s_tv, v, -1, sc,
                                          unused);
                  if (sc > -INFINITY) best_merge(br, Best{sc, v});
                }
              }
            }
          }
        } else {
          br = Best{-INFINITY, -1};  // no candidate with p > q among 2 x 256 tokens: stream the share
        }
      }
    }
    // Every load of the kU units a thread takes per iteration is issued before
    // any is used: one memory round trip per iteration for up to KB draft
    // categories (further categories in batches of KB).
    constexpr int kU = KB == 1 ? 2 : 1;
    for (int64_t u0 = ua; stream && u0 < u1; u0 += kU * kThreads) {
      uint4 tv[kU], gw[kU][VEC ? E / 4 : 1], dv[kU][KB];
      float xs[kU], gs[kU], ds[kU][KB];
#pragma unroll
      for (int h = 0; h < kU; ++h) {
        const int64_t u = u0 + h * kThreads;
        if (u >= u1) break;
        if constexpr (VEC) {
          tv[h] = ldg16(reinterpret_cast<const uint4*>(trow) + u);
#pragma unroll
          for (int c = 0; c < E / 4; ++c) gw[h][c] = ldg16(reinterpret_cast<const uint4*>(grow + u * E) + c);
        } else {
          xs[h] = Elem<DT>::at(trow, u);
          gs[h] = __ldg(grow + u);
        }
        if (resid) {
#pragma unroll
          for (int z = 0; z < KB; ++z)
            if (z < K) {
              if constexpr (VEC) dv[h][z] = ldg16(reinterpret_cast<const uint4*>(dbase + z * dstride) + u);
              else ds[h][z] = Elem<DT>::at(dbase + z * dstride, u);
            }
        }
      }
#pragma unroll
      for (int h = 0; h < kU; ++h) {
        const int64_t u = u0 + h * kThreads;
        if (u >= u1) break;
        float xt[E], gv[E], q[E];
        if constexpr (VEC) {
          Elem<DT>::unpack(tv[h], xt);
#pragma unroll
          for (int c = 0; c < E / 4; ++c) {
            gv[4 * c] = __uint_as_float(gw[h][c].x); gv[4 * c + 1] = __uint_as_float(gw[h][c].y);
            gv[4 * c + 2] = __uint_as_float(gw[h][c].z); gv[4 * c + 3] = __uint_as_float(gw[h][c].w);
          }
        } else {
          xt[0] = xs[h];
          gv[0] = gs[h];
        }
#pragma unroll
        for (int e = 0; e < E; ++e) {
          q[e] = 0.f;
          if (!resid && kept<TP>(s_tk, s_tv, 0, xt[e], u * E + e)) {  // bonus draw (after a rejection the bonus
            // rule is only a rare fallback, below)
            const Best c{static_cast<double>(xt[e]) * invT + static_cast<double>(gv[e]), static_cast<int>(u * E + e)};
            if (c.score > bb.score) bb = c;
          }
        }
        if (resid) {
#pragma unroll
          for (int z = 0; z < KB; ++z)
            if (z < K) {
              float xd[E];
              if constexpr (VEC) Elem<DT>::unpack(dv[h][z], xd);
              else xd[0] = ds[h][z];
              const float cz = s_c[1 + z], mz = s_mm[1 + z];
#pragma unroll
              for (int e = 0; e < E; ++e)
                q[e] = fmaf(cz, kept<TP>(s_tk, s_tv, 1 + z, xd[e], u * E + e) ? ex2((xd[e] - mz) * k) : 0.f, q[e]);
            }
          for (int z0 = KB; z0 < K; z0 += KB) {  // K > KB: further round trips
#pragma unroll
            for (int z = 0; z < KB; ++z)
              if (z0 + z < K) {
                if constexpr (VEC) dv[h][z] = ldg16(reinterpret_cast<const uint4*>(dbase + (z0 + z) * dstride) + u);
                else ds[h][z] = Elem<DT>::at(dbase + (z0 + z) * dstride, u);
              }
#pragma unroll
            for (int z = 0; z < KB; ++z)
              if (z0 + z < K) {
                float xd[E];
                if constexpr (VEC) Elem<DT>::unpack(dv[h][z], xd);
                else xd[0] = ds[h][z];
                const float cz = s_c[1 + z0 + z], mz = s_mm[1 + z0 + z];
#pragma unroll
                for (int e = 0; e < E; ++e)
                  q[e] = fmaf(cz, kept<TP>(s_tk, s_tv, 1 + z0 + z, xd[e], u * E + e) ? ex2((xd[e] - mz) * k) : 0.f,
                              q[e]);
              }
          }
#pragma unroll
          for (int e = 0; e < E; ++e) {
            const float r = fmaf(kept<TP>(s_tk, s_tv, 0, xt[e], u * E + e) ? ex2((xt[e] - mt) * k) : 0.f, ct, -q[e]);
            if (r > 0.f) {
              const Best c{static_cast<double>(lg2(r) * kLn2) + static_cast<double>(gv[e]), static_cast<int>(u * E + e)};
              if (c.score > br.score) br = c;
            }
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

  // ---- 4. the last of the request's P blocks writes its terminal token. The
  //         block barrier orders every thread's outputs and keys before thread
  //         0's ticket, whose gpu-scope release publishes them and whose
  //         acquire (in the last block) makes the other blocks' keys visible.
  __syncthreads();
  if (tid == 0) {
    s_last = ticket_acq_rel(a.tickets + b) == a.P - 1;
    s_fail = 0;
  }
  __syncthreads();
  if (!s_last) return;
  if (tid == 0) {
    s_scan = 0;
    if (flags == 0) {
      const int j = s_j;
      const unsigned long long kr = __ldcg(a.keys + 2 * b), kb = __ldcg(a.keys + 2 * b + 1);
      if (j < ell && !kr) {
        s_scan = 1;  // rounding left no p > q after a rejection: bonus rule on row j, below
      } else {
        const int term = j < ell ? key_token(kr) : key_token(kb);
        if (term >= 0) out[j] = term;
        else s_fail = 1;
      }
    }
    a.keys[2 * b] = 0ull;
    a.keys[2 * b + 1] = 0ull;
    a.tickets[b] = 0;
  }
  __syncthreads();
  if (s_scan) {  // rare: this block takes argmax_v x_j(v) / T + g(v) over the whole row
    const int j = s_j;
    const double invT = 1.0 / static_cast<double>(a.T);
    const char* trow = static_cast<const char*>(a.target) + (toff + j) * V * Elem<DT>::kBytes;
    const float* grow = a.g + (static_cast<int64_t>(b) * (L + 1) + j) * V;
    Best bb{-INFINITY, -1};
    for (int64_t v = tid; v < V; v += kThreads) {
      const float x = Elem<DT>::at(trow, v);
      if (!kept<TP>(s_tk, s_tv, 0, x, v)) continue;  // filtered: row j's nucleus
      const Best c{static_cast<double>(x) * invT + static_cast<double>(__ldg(grow + v)), static_cast<int>(v)};
      if (c.score > bb.score) bb = c;
    }
    warp_best(bb);
    if (lane == 0) s_best[tid >> 5] = bb;
    __syncthreads();
    if (tid == 0) {
      Best t = s_best[0];
      for (int w = 1; w < kWarps; ++w) best_merge(t, s_best[w]);
      if (t.idx >= 0) out[j] = t.idx;
      else s_fail = 1;
    }
    __syncthreads();
  }
  if (s_fail) {  // no finite candidate in the terminal row: the request fails as a whole
    for (int i = tid; i <= L; i += kThreads) out[i] = -1;
    if (tid == 0) {
      a.accept_len[b] = -1;
      atomicOr(a.status, kFlagNonFinite);
    }
  }
}

template <int DT, bool VEC, bool TP>
static auto accept_kernel(int K) {
  return K == 1 ? k_accept_sample<DT, VEC, 1, TP> : k_accept_sample<DT, VEC, 4, TP>;
}

template <bool TP>
static auto accept_kernel(int dtype, bool vec, int K) {
  if (dtype == 0) return vec ? accept_kernel<0, true, TP>(K) : accept_kernel<0, false, TP>(K);
  return vec ? accept_kernel<1, true, TP>(K) : accept_kernel<1, false, TP>(K);
}

int accept_blocks_per_sm(int dtype, bool vec, int K, bool topp) {
  int occ = 0;
  const cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(
      &occ, topp ? accept_kernel<true>(dtype, vec, K) : accept_kernel<false>(dtype, vec, K), kThreads, 0);
  return (e == cudaSuccess && occ > 0) ? occ : 1;
}

cudaError_t launch_accept_sample(const VerifyArgs& a, int dtype, bool vec, cudaStream_t st) {
  const float k = static_cast<float>(1.4426950408889634 / static_cast<double>(a.T));
  auto kernel = a.topp ? accept_kernel<true>(dtype, vec, a.K) : accept_kernel<false>(dtype, vec, a.K);
  return launch_pdl(kernel, dim3(a.P, a.B), dim3(kThreads), 0, st, a, k);
}

}  // namespace specv
