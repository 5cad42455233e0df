// One persistent kernel per verify step: the fused temperature softmax of
// the verify window, the accept decisions and the terminal Gumbel-max draws.
//
// Method: speculative sampling with rejection correction over independent or
// latent-mixture drafts ("DBLAST: Dependent Block Drafting for Stochastic
// Speculative Decoding", Pith review, "Assumptions" and "What carries the
// argument", Eq. 5); fixed-address workspaces that carry variable
// boundaries through verification ("DScale: Scaling Block-Diffusion
// Speculative Decoding with Adaptive Verification", Abstract).
//
// Schedule. One block per SM. A global work queue lists, in order,
//   S_0, S_1, T_0, S_2, T_1, ..., S_{B-1}, T_{B-2}, T_{B-1}
// where S_b are the 32 KB chunks of request b's window rows (statistics
// items) and T_b the chunks of its terminal row (terminal items). Blocks
// take items with an atomic counter. The block that completes S_b's last
// chunk merges b's partials, takes the accept decisions (fp64, one warp) and
// publishes them; T_b is queued behind S_{b+1}, so by the time a block
// takes a T_b item the decision is usually there, and requests finish in a
// pipeline while later requests still stream.
//
// Inside a block, one producer warp moves each item from HBM into a 6-stage
// ring of 32 KB shared-memory stages with 1-D bulk copies (cp.async.bulk,
// completion on an mbarrier); 16 consumer warps fold the statistics or score
// the terminal elements and release the stage.
//
// Every wait (stage barriers, the decision flag) is bounded by %globaltimer;
// on expiry the block raises SPEC_DEV_TIMEOUT, stops, drains its own copies
// and exits. Nothing waits on work that has not been taken by a running
// block, so the bound is never reached in a correct run.
#include <algorithm>

#include "common.cuh"
#include "decide.cuh"
#include "internal.h"

namespace specv {

constexpr int kCW = 16;              // consumer warps
constexpr int kCT = kCW * 32;        // consumer threads
constexpr int kFT = kCT + 32;        // + one producer warp
constexpr int kFlagTimeout = 16;
constexpr uint64_t kWaitNs = 1000000000ull;

enum : int { kItemStats = 0, kItemTerm = 1, kItemTermNoop = 2, kItemEnd = 3, kItemFlush = 4 };

struct __align__(16) StageMeta {
  int kind, b, n, slot;  // n: 16 B units (statistics) or elements (terminal); slot: partial index or chunk p
  int row, tok;          // statistics: window row; token offset inside the chunk (elements) or -1
  int j, flags, ell, v0;  // terminal: decision, first element of the chunk
  float ct, mt;
  float cz[kMaxK], mz[kMaxK];
};

// ------------------------------------------------------------ PTX helpers

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ uint64_t gtime() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}
// Add expected transaction bytes to the current phase without arriving.
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Wait for the phase of the given parity to complete, until `deadline`.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint64_t deadline) {
  while (!mbar_test(bar, parity))
    if (gtime() > deadline) return false;
  return true;
}
// 1-D bulk copy global -> this block's shared memory, completing on `bar`.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_addr(dst)),
               "l"(src), "r"(bytes), "r"(smem_addr(bar))
               : "memory");
}
__device__ __forceinline__ int ld_acquire(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release(int* p, int v) {
  asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
// Named barrier over the consumer warps only.
__device__ __forceinline__ void consumers_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kCT) : "memory"); }

// ------------------------------------------------------------- queue layout

// Queue order with lag kLag: S_0 .. S_{kLag-1}, then S_k, T_{k-kLag} for
// k = kLag .. B-1, then the remaining T. Returns the segment positions.
constexpr int kLag = 2;
__device__ __forceinline__ int seg_pos_stats(int b) { return b < kLag ? b : kLag + 2 * (b - kLag); }
__device__ __forceinline__ int seg_pos_term(int b, int B) { return b + kLag <= B - 1 ? kLag + 2 * b + 1 : B + b; }

__device__ __forceinline__ int atom_add_acq_rel(int* p, int v) {
  int old;
  asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

// --------------------------------------------------------------- the kernel

enum : int { kActNone = 0, kActDecide = 1, kActFinal = 2 };
constexpr int kStash = 8;

struct FusedShared {
  StageMeta meta[kFusedStages];
  uint64_t full[kFusedStages];
  uint64_t empty[kFusedStages];
  float d_xg[kMaxRows], d_m[kMaxRows], d_s[kMaxRows];
  int d_x[kMaxL];
  float2 red[kCW];
  Best redr[kCW], redb[kCW];
  int scan_tmp[kFT / 32 + 1];
  int epoch, abort_, flags;
  int act, act_b, act_j, act_ell, act_flags;  // action of the previous stage, run at the next stage's top
};

template <int DT>
__device__ __forceinline__ const char* window_row(const FusedArgs& a, const int* toff, int b, int ell, int q) {
  constexpr int64_t esz = Elem<DT>::kBytes;
  if (q < ell) return static_cast<const char*>(a.target) + (static_cast<int64_t>(toff[b]) + q) * a.V * esz;
  const int q2 = q - ell, z = q2 / ell, i = q2 - z * ell;
  return static_cast<const char*>(a.draft) + ((static_cast<int64_t>(b) * a.K + z) * a.L + i) * a.V * esz;
}

template <int DT>
__global__ void __launch_bounds__(kFT, 1) k_verify_fused(FusedArgs a) {
  constexpr int E = Elem<DT>::kPerVec;
  constexpr int ES = Elem<DT>::kBytes;
  extern __shared__ __align__(128) unsigned char smem[];
  unsigned char* stages = smem;
  FusedShared& sh = *reinterpret_cast<FusedShared*>(smem + kFusedStages * kFusedStageBytes);
  int* rowoff = reinterpret_cast<int*>(&sh + 1);  // [B + 1] window row offset of each request
  int* segoff = rowoff + a.B + 1;                  // [2B + 1] queue offset of each segment
  int* seginfo = segoff + 2 * a.B + 1;             // [2B] (b << 1) | is_terminal
  int* toff = seginfo + 2 * a.B;                   // [B] target row of (b, 0)

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int B = a.B, K = a.K;
  pdl_wait();
  const uint64_t deadline = gtime() + kWaitNs;

  // ---- setup: request lengths -> row offsets -> queue segments
  for (int b = tid; b < B; b += kFT) {
    int l = a.vlen ? a.vlen[b] : a.L;
    if (l < 0 || l > a.L) l = 0;  // flagged where the request is decided
    rowoff[b] = (K + 1) * l;
    toff[b] = a.row_off ? a.row_off[b] : b * (a.L + 1);
    seginfo[seg_pos_stats(b)] = b << 1;
    seginfo[seg_pos_term(b, B)] = (b << 1) | 1;
  }
  __syncthreads();
  const int total_rows = block_exclusive_scan<kFT>(rowoff, B, sh.scan_tmp);
  if (tid == 0) rowoff[B] = total_rows;
  for (int q = tid; q < 2 * B; q += kFT) {
    const int b = seginfo[q] >> 1;
    const int nrows = (b + 1 < B ? rowoff[b + 1] : total_rows) - rowoff[b];
    segoff[q] = (seginfo[q] & 1) ? a.Pt : nrows * a.cpr;
  }
  __syncthreads();
  const int total_items = block_exclusive_scan<kFT>(segoff, 2 * B, sh.scan_tmp);
  if (tid == 0) {
    segoff[2 * B] = total_items;
    sh.epoch = __ldcg(a.ctl);
    sh.abort_ = 0;
    sh.act = kActNone;
    for (int s = 0; s < kFusedStages; ++s) {
      mbar_init(&sh.full[s], 1);
      mbar_init(&sh.empty[s], kCW);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  pdl_trigger();
  const int epoch = sh.epoch;
  volatile int* abort_flag = &sh.abort_;

  if (warp == kCW) {
    // ================================================================ producer
    if (lane == 0) {
      int s = 0;
      uint32_t round = 0;
      int filled[kFusedStages];  // round in which each stage was last armed, -1 if never
#pragma unroll
      for (int t = 0; t < kFusedStages; ++t) filled[t] = -1;
      int stash_b[kStash], stash_p[kStash], nstash = 0;  // terminal items waiting for their decision
      int next = atomicAdd(a.ctl + 1, 1);
      bool flushed = false;  // a flush stage is out since the last item
      // Before waiting for a decision, hand the consumers an empty "flush" stage:
      // they run the completion check they deferred from their last stage, which
      // may be the very decision this block waits for.
      auto flush = [&]() -> bool {
        if (flushed) return true;
        if (!mbar_wait(&sh.empty[s], (round & 1) ^ 1, deadline)) return false;
        filled[s] = static_cast<int>(round);
        sh.meta[s].kind = kItemFlush;
        mbar_arrive(&sh.full[s]);
        if (++s == kFusedStages) {
          s = 0;
          ++round;
        }
        flushed = true;
        return true;
      };
      for (;;) {
        // ---- pick an item: a stashed terminal item whose decision is out, else the queue
        int kind = -1, b = 0, local = 0;
        bool end = false;
        if (nstash > 0 && ld_acquire(a.dready + stash_b[0]) == epoch + 1) {
          kind = kItemTerm;
          b = stash_b[0];
          local = stash_p[0];
          for (int t = 1; t < nstash; ++t) { stash_b[t - 1] = stash_b[t]; stash_p[t - 1] = stash_p[t]; }
          --nstash;
        } else if (next < total_items && !*abort_flag) {
          const int i = next;
          next = atomicAdd(a.ctl + 1, 1);
          int lo = 0, hi = 2 * B - 1;  // segment holding item i
          while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (segoff[mid] <= i) lo = mid; else hi = mid - 1;
          }
          b = seginfo[lo] >> 1;
          kind = (seginfo[lo] & 1) ? kItemTerm : kItemStats;
          local = i - segoff[lo];
          if (kind == kItemTerm && rowoff[b + 1] > rowoff[b] && ld_acquire(a.dready + b) != epoch + 1) {
            if (nstash < kStash) {
              stash_b[nstash] = b;
              stash_p[nstash] = local;
              ++nstash;
              continue;
            }
            if (!flush()) { atomicOr(a.status, kFlagTimeout); *abort_flag = 1; }
            while (ld_acquire(a.dready + b) != epoch + 1 && !*abort_flag)
              if (gtime() > deadline) { atomicOr(a.status, kFlagTimeout); *abort_flag = 1; }
          }
        } else if (nstash > 0 && !*abort_flag) {
          // queue exhausted: wait for the oldest stashed decision
          if (!flush() || gtime() > deadline) { atomicOr(a.status, kFlagTimeout); *abort_flag = 1; }
          continue;
        } else {
          end = true;
        }
        if (*abort_flag) end = true;
        // ---- a free stage
        if (!mbar_wait(&sh.empty[s], (round & 1) ^ 1, deadline)) {
          atomicOr(a.status, kFlagTimeout);
          *abort_flag = 1;
          break;
        }
        StageMeta& mt = sh.meta[s];
        unsigned char* buf = stages + s * kFusedStageBytes;
        filled[s] = static_cast<int>(round);
        flushed = false;
        if (end) {
          mt.kind = kItemEnd;
          mbar_arrive(&sh.full[s]);
          break;
        }
        const int ell = (rowoff[b + 1] - rowoff[b]) / (K + 1);
        if (kind == kItemStats) {
          const int q = local / a.cpr, c = local - q * a.cpr;
          const int64_t u0 = c * a.Vu / a.cpr, u1 = (c + 1) * a.Vu / a.cpr;
          const uint32_t bytes = static_cast<uint32_t>(u1 - u0) * 16u;
          // order: expected bytes, copy, metadata, then the producer's arrival
          // (release): the phase completes only after all four
          mbar_expect_tx(&sh.full[s], bytes);
          bulk_load(buf, window_row<DT>(a, toff, b, ell, q) + u0 * 16, bytes, &sh.full[s]);
          mt.kind = kItemStats;
          mt.b = b;
          mt.n = static_cast<int>(u1 - u0);
          mt.row = rowoff[b] + q;
          mt.slot = mt.row * a.cpr + c;
          mbar_arrive(&sh.full[s]);
        } else {
          const int p = local;
          int j = 0, flags = 0;
          if (ell == 0) {
            const bool bad_len = a.vlen && (a.vlen[b] < 0 || a.vlen[b] > a.L);
            flags = bad_len ? kFlagVerifyLen : 0;  // nothing to test: a bonus draw from row 0
          } else {
            j = __ldcg(&a.dec[b].j);
            flags = __ldcg(&a.dec[b].flags);
          }
          mt.b = b;
          mt.slot = p;
          mt.j = j;
          mt.flags = flags;
          mt.ell = ell;
          if (flags) {
            mt.kind = kItemTermNoop;
            mbar_arrive(&sh.full[s]);
          } else {
            const int64_t g0 = p * a.Vq / a.Pt, g1 = (p + 1) * a.Vq / a.Pt;
            const int n = static_cast<int>((g1 - g0) * 8);
            const int64_t v0 = g0 * 8;
            const bool resid = j < ell;
            const uint32_t seg = static_cast<uint32_t>(n) * ES;
            const uint32_t bytes = seg * (resid ? K + 1 : 1) + static_cast<uint32_t>(n) * 4u;
            mbar_expect_tx(&sh.full[s], bytes);
            const int64_t trow = static_cast<int64_t>(toff[b]) + j;
            bulk_load(buf, static_cast<const char*>(a.target) + (trow * a.V + v0) * ES, seg, &sh.full[s]);
            if (resid)
              for (int z = 0; z < K; ++z)
                bulk_load(buf + seg * (1 + z),
                          static_cast<const char*>(a.draft) +
                              (((static_cast<int64_t>(b) * K + z) * a.L + j) * a.V + v0) * ES,
                          seg, &sh.full[s]);
            bulk_load(buf + seg * (K + 1), a.g + (static_cast<int64_t>(b) * (a.L + 1) + j) * a.V + v0,
                      static_cast<uint32_t>(n) * 4u, &sh.full[s]);
            mt.kind = kItemTerm;
            mt.n = n;
            mt.v0 = static_cast<int>(v0);
            if (resid) {
              mt.ct = __ldcg(&a.dec[b].ct);
              mt.mt = __ldcg(&a.dec[b].mt);
              for (int z = 0; z < K; ++z) {
                mt.cz[z] = __ldcg(&a.dec[b].cz[z]);
                mt.mz[z] = __ldcg(&a.dec[b].mz[z]);
              }
            }
            mbar_arrive(&sh.full[s]);
          }
        }
        if (++s == kFusedStages) {
          s = 0;
          ++round;
        }
      }
      // drain: wait until every copy this block armed has landed
#pragma unroll
      for (int t = 0; t < kFusedStages; ++t)
        if (filled[t] >= 0 && !mbar_wait(&sh.full[t], filled[t] & 1, deadline + kWaitNs))
          atomicOr(a.status, kFlagTimeout);
    }
    __syncwarp();
  } else {
    // ================================================================ consumers
    const int ctid = tid;
    int s = 0;
    uint32_t round = 0;
    // lane 0 of warp 0: the completion count of the previous stage, checked one stage later
    int pend_kind = -1, pend_b = 0, pend_ret = 0, pend_j = 0, pend_ell = 0, pend_flags = 0;
    for (;;) {
      // every consumer waits (bounded) for the stage; a failure anywhere makes
      // all consumer warps leave together, so the named barriers stay matched
      if (!mbar_wait(&sh.full[s], round & 1, deadline)) {
        atomicOr(a.status, kFlagTimeout);
        *abort_flag = 1;
      }
      if (ctid == 0) {
        int act = kActNone;
        if (pend_kind == kItemStats && pend_ret + 1 == (rowoff[pend_b + 1] - rowoff[pend_b]) * a.cpr) act = kActDecide;
        if ((pend_kind == kItemTerm || pend_kind == kItemTermNoop) && pend_ret + 1 == a.Pt) act = kActFinal;
        sh.act = act;
        sh.act_b = pend_b;
        sh.act_j = pend_j;
        sh.act_ell = pend_ell;
        sh.act_flags = pend_flags;
        sh.flags = 0;
        pend_kind = -1;
      }
      consumers_sync();
      if (*abort_flag) break;
      const int act = sh.act, ab = sh.act_b;
      if (act == kActDecide) {
        // ---- decide request ab: merge its rows' partials and gather the drafted-token
        // logits, then one warp takes the accept decisions in fp64
        __threadfence();
        const int base = rowoff[ab], nrows = rowoff[ab + 1] - rowoff[ab];
        const int ell = nrows / (K + 1);
        if (ctid < ell) {
          const int x = __ldg(a.tokens + static_cast<int64_t>(ab) * a.L + ctid);
          if (x < 0 || x >= a.V) atomicOr(&sh.flags, kFlagTokenRange);
          sh.d_x[ctid] = (x < 0 || x >= a.V) ? 0 : x;
        }
        consumers_sync();
        for (int q = ctid; q < nrows; q += kCT) {
          const int pos = q < ell ? q : (q - ell) % ell;
          const float xq = Elem<DT>::at(window_row<DT>(a, toff, ab, ell, q), sh.d_x[pos]);
          float mm = -INFINITY, ss = 0.f;
          const float2* pp = a.part + static_cast<int64_t>(base + q) * a.cpr;
          for (int c = 0; c < a.cpr; c += 8) {  // 8 independent loads in flight per round trip
            float2 pr[8];
#pragma unroll
            for (int t = 0; t < 8; ++t) pr[t] = c + t < a.cpr ? __ldcg(pp + c + t) : make_float2(-INFINITY, 0.f);
#pragma unroll
            for (int t = 0; t < 8; ++t) ms_merge(mm, ss, pr[t].x, pr[t].y, a.k);
          }
          sh.d_m[q] = mm;
          sh.d_s[q] = ss;
          sh.d_xg[q] = xq;
          if (!isfinite(mm) || !isfinite(ss)) atomicOr(&sh.flags, kFlagNonFinite);
        }
        consumers_sync();
        if (warp == 0) {
          int flags = sh.flags;
          DecideOut o = {};
          o.j = -1;
          if (!flags) {
            const DecideIn in{sh.d_xg, sh.d_m, sh.d_s, sh.d_x, ell, K, a.L, a.T};
            o = decide_warp(in, a.u + static_cast<int64_t>(ab) * a.L,
                            a.mix_w ? a.mix_w + static_cast<int64_t>(ab) * K : nullptr);
            if (o.bad) flags |= kFlagNonFinite;
          }
          if (lane == 0) {
            Decision& d = a.dec[ab];
            d.j = o.j;
            d.flags = flags;
            d.ell = ell;
            d.ct = o.ct;
            d.mt = o.mt;
            for (int z = 0; z < kMaxK; ++z) {
              d.cz[z] = z < K ? o.cz[z] : 0.f;
              d.mz[z] = z < K ? o.mz[z] : 0.f;
            }
            a.req_cnt[ab] = 0;
            __threadfence();
            st_release(a.dready + ab, epoch + 1);
          }
        }
      } else if (act == kActFinal && warp == 0) {
        // ---- the last terminal chunk of request ab: merge the chunk partials, write the outputs
        __threadfence();
        const int j = sh.act_j, ell = sh.act_ell, flags = sh.act_flags;
        Best r{-INFINITY, -1}, o{-INFINITY, -1};
        for (int c = lane; c < a.Pt; c += 32) {
          const TermPart* tp = a.tpart + static_cast<int64_t>(ab) * a.Pt + c;
          best_merge(r, Best{__ldcg(&tp->res_score), __ldcg(&tp->res_idx)});
          best_merge(o, Best{__ldcg(&tp->bon_score), __ldcg(&tp->bon_idx)});
        }
        warp_best(r);
        warp_best(o);
        const int t = flags == 0 ? ((j < ell && r.idx >= 0) ? r.idx : o.idx) : -1;
        const bool ok = flags == 0 && t >= 0;
        int32_t* out = a.out_tokens + static_cast<int64_t>(ab) * (a.L + 1);
        for (int i = lane; i <= a.L; i += 32)
          out[i] = !ok ? -1 : (i < j ? __ldg(a.tokens + static_cast<int64_t>(ab) * a.L + i) : (i == j ? t : -1));
        if (lane == 0) {
          a.accept_len[ab] = ok ? j : -1;
          if (flags) atomicOr(a.status, flags);
          else if (!ok) atomicOr(a.status, kFlagNonFinite);
          a.tterm[ab] = 0;
        }
      }
      const StageMeta& mt = sh.meta[s];
      const int kind = mt.kind;
      if (kind == kItemEnd) break;
      const unsigned char* buf = stages + s * kFusedStageBytes;
      const int b = mt.b;
      if (kind == kItemFlush) {
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.empty[s]);
      } else if (kind == kItemStats) {
        const uint4* sv = reinterpret_cast<const uint4*>(buf);
        const int n = mt.n;
        const int slot = mt.slot;
        float m = -INFINITY, sum = 0.f;
        if (ctid + 3 * kCT < n) {
          const uint4 v[4] = {sv[ctid], sv[ctid + kCT], sv[ctid + 2 * kCT], sv[ctid + 3 * kCT]};
          fold_vectors<DT, 4>(v, m, sum, a.k);
        } else {
          for (int u = ctid; u < n; u += kCT) {
            const uint4 v[1] = {sv[u]};
            fold_vectors<DT, 1>(v, m, sum, a.k);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.empty[s]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
          const float s2 = __shfl_xor_sync(0xffffffffu, sum, o);
          ms_merge(m, sum, m2, s2, a.k);
        }
        if (lane == 0) sh.red[warp] = make_float2(m, sum);
        consumers_sync();
        if (warp == 0) {
          float2 v = lane < kCW ? sh.red[lane] : make_float2(-INFINITY, 0.f);
          m = v.x;
          sum = v.y;
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) {
            const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
            const float s2 = __shfl_xor_sync(0xffffffffu, sum, o);
            ms_merge(m, sum, m2, s2, a.k);
          }
          if (lane == 0) {
            a.part[slot] = make_float2(m, sum);
            pend_ret = atom_add_acq_rel(a.req_cnt + b, 1);  // read at the next stage's top
            pend_kind = kItemStats;
            pend_b = b;
          }
        }
      } else {
        // ---- terminal chunk: best residual and bonus scores over [v0, v0 + n)
        Best br{-INFINITY, -1}, bb{-INFINITY, -1};
        const int j = mt.j, ell = mt.ell, flags = mt.flags, p = mt.slot;
        if (kind == kItemTerm) {
          const int n = mt.n, v0 = mt.v0;
          const bool resid = j < ell;
          const double invT = 1.0 / static_cast<double>(a.T);
          const float ct = mt.ct, mtt = mt.mt;
          const int seg = n * ES;
          const float* gs = reinterpret_cast<const float*>(buf + seg * (K + 1));
          for (int u = ctid; u < n / E; u += kCT) {
            float xt[E], gv[E], q[E];
            Elem<DT>::unpack(reinterpret_cast<const uint4*>(buf)[u], xt);
#pragma unroll
            for (int h = 0; h < E / 4; ++h) {
              const float4 w = reinterpret_cast<const float4*>(gs + u * E)[h];
              gv[4 * h] = w.x; gv[4 * h + 1] = w.y; gv[4 * h + 2] = w.z; gv[4 * h + 3] = w.w;
            }
#pragma unroll
            for (int e = 0; e < E; ++e) {
              const Best c{static_cast<double>(xt[e]) * invT + static_cast<double>(gv[e]), v0 + u * E + e};
              if (c.score > bb.score) bb = c;
              q[e] = 0.f;
            }
            if (resid) {
              for (int z = 0; z < K; ++z) {
                float xd[E];
                Elem<DT>::unpack(reinterpret_cast<const uint4*>(buf + seg * (1 + z))[u], xd);
                const float cz = mt.cz[z], mz = mt.mz[z];
#pragma unroll
                for (int e = 0; e < E; ++e) q[e] = fmaf(cz, ex2((xd[e] - mz) * a.k), q[e]);
              }
#pragma unroll
              for (int e = 0; e < E; ++e) {
                const float r = ex2((xt[e] - mtt) * a.k) * ct - q[e];
                if (r > 0.f) {
                  const Best c{static_cast<double>(lg2(r) * kLn2) + static_cast<double>(gv[e]), v0 + u * E + e};
                  if (c.score > br.score) br = c;
                }
              }
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.empty[s]);
        warp_best(br);
        warp_best(bb);
        if (lane == 0) {
          sh.redr[warp] = br;
          sh.redb[warp] = bb;
        }
        consumers_sync();
        if (warp == 0) {
          br = lane < kCW ? sh.redr[lane] : Best{-INFINITY, -1};
          bb = lane < kCW ? sh.redb[lane] : Best{-INFINITY, -1};
          warp_best(br);
          warp_best(bb);
          if (lane == 0) {
            a.tpart[static_cast<int64_t>(b) * a.Pt + p] = TermPart{br.score, bb.score, br.idx, bb.idx, {0, 0}};
            pend_ret = atom_add_acq_rel(a.tterm + b, 1);  // read at the next stage's top
            pend_kind = kind;
            pend_b = b;
            pend_j = j;
            pend_ell = ell;
            pend_flags = flags;
          }
        }
      }
      if (++s == kFusedStages) {
        s = 0;
        ++round;
      }
    }
  }

  // ---- exit: the last block out resets the queue and advances the epoch
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    if (atomicAdd(a.ctl + 2, 1) == static_cast<int>(gridDim.x) - 1) {
      a.ctl[1] = 0;
      a.ctl[2] = 0;
      __threadfence();
      a.ctl[0] = epoch + 1;
    }
  }
}

// ------------------------------------------------------------------- host

int fused_cpr(int64_t V, int dtype) {
  const int64_t Vu = V * (dtype == 0 ? 4 : 2) / 16;
  const int64_t cap = kFusedStageBytes / 16;
  return static_cast<int>(std::max<int64_t>(1, (Vu + cap - 1) / cap));
}

int fused_pt(int64_t V, int dtype, int K) {
  const int64_t es = dtype == 0 ? 4 : 2;
  const int64_t per_group = 8 * (es * (K + 1) + 4);  // bytes of 8 elements of every operand
  const int64_t groups = kFusedStageBytes / per_group;
  const int64_t Vq = V / 8;
  return static_cast<int>(std::max<int64_t>(1, (Vq + groups - 1) / groups));
}

size_t fused_smem_bytes(int B) {
  return static_cast<size_t>(kFusedStages) * kFusedStageBytes + sizeof(FusedShared) +
         static_cast<size_t>(6 * B + 2) * sizeof(int);
}

cudaError_t launch_fused(const FusedArgs& a, int dtype, int grid, cudaStream_t st) {
  const size_t smem = fused_smem_bytes(a.B);
  void (*kern)(FusedArgs) = dtype == 0 ? k_verify_fused<0> : k_verify_fused<1>;
  const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, dim3(grid), dim3(kFT), smem, st, a);
}

}  // namespace specv
