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
// Schedule. One block per SM (the grid is the SM count and each block
// takes most of the shared memory, so all blocks are resident together).
//  Phase 1: the window's rows, flattened into 16-byte units, are split
//   evenly over the blocks; each block streams its share through a ring of
//   six 32 KB shared-memory stages filled by 1-D bulk copies
//   (cp.async.bulk, completion on an mbarrier) issued by one producer warp.
//   16 consumer warps fold every stage into per-thread online
//   (max, sum of exp) statistics and reduce across the block only where the
//   block's share of a row ends, writing one partial per (row, block).
//  Then every block adds its row pieces to each request's counter; the block
//   owning a request's last unit waits for the request's full count, merges
//   its partials and takes the accept decisions (fp64, one warp).
//  Phase 2: the B x Pt chunks of the terminal rows are dealt round-robin to
//   the blocks; each waits for its request's decision, streams target, draft
//   and Gumbel chunk, scores it, and the last chunk of a request writes the
//   outputs.
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
// try_wait with a suspend-time hint: the thread sleeps in hardware until the
// phase completes or about `ns` nanoseconds pass, so waiting warps take no
// issue slots from the producer.
__device__ __forceinline__ bool mbar_test_sleep(uint64_t* bar, uint32_t parity, uint32_t ns) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity), "r"(ns)
      : "memory");
  return ok != 0;
}
// Wait for the phase of the given parity to complete, until `deadline`.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint64_t deadline) {
  if (mbar_test(bar, parity)) return true;
  while (!mbar_test_sleep(bar, parity, 20000u))
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
__device__ __forceinline__ unsigned long long ld_acquire_u64(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release(int* p, int v) {
  asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
// Order-preserving 64-bit key of a terminal candidate: the fp64 score with
// its lowest 20 bits replaced by (2^20 - 1 - token), so that an unsigned max
// picks the highest score and, among equal scores, the lowest token. 0 means
// "no candidate". Needs V <= 2^20; the score keeps 32 significant bits.
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
// owner of unit e in the even split, without a 64-bit integer division
__device__ __forceinline__ int64_t owner_of(int64_t e, int64_t N, int64_t G) {
  const int64_t num = (e + 1) * G - 1;
  int64_t q = static_cast<int64_t>(static_cast<double>(num) / static_cast<double>(N));
  while (q > 0 && q * N > num) --q;
  while ((q + 1) * N <= num) ++q;
  return q;
}
// Named barrier over the consumer warps only.
__device__ __forceinline__ void consumers_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kCT) : "memory"); }

// --------------------------------------------------------------- the kernel

enum : int { kItemStats = 0, kItemTerm = 1, kItemTermNoop = 2, kItemEnd = 3, kItemPhaseEnd = 4 };

struct __align__(16) StageMeta {
  int kind, b, n, slot;   // n: 16 B units (statistics) or elements (terminal); slot: partial index or chunk p
  int row, tok, seg_end;  // statistics: window row; drafted token inside the chunk (element) or -1; last chunk of the segment
  int seg_units;          // statistics, last chunk: units of this block's segment of the row
  int j, flags, ell, v0;  // terminal: decision, first element of the chunk
  float ct, mt;
  float cz[kMaxK], mz[kMaxK];
};

struct FusedShared {
  StageMeta meta[kFusedStages];
  uint64_t full[kFusedStages];
  uint64_t empty[kFusedStages];
  float d_xg[kMaxRows], d_m[kMaxRows], d_s[kMaxRows];
  int d_x[kMaxL];
  float2 red[kCW];
  Best redr[kCW], redb[kCW];
  int scan_tmp[kFT / 32 + 1];
  uint64_t dbar, ddone;  // decision: rows merged (16 warps), decision published (warp 0)
  int epoch, abort_, flags, last;
  int rtok[64];  // drafted token of this block's first 64 window rows
};

template <int DT>
__device__ __forceinline__ const char* window_row(const FusedArgs& a, const int* toff, int b, int ell, int q) {
  constexpr int64_t esz = Elem<DT>::kBytes;
  if (q < ell) return static_cast<const char*>(a.target) + (static_cast<int64_t>(toff[b]) + q) * a.V * esz;
  const int q2 = q - ell, z = q2 / ell, i = q2 - z * ell;
  return static_cast<const char*>(a.draft) + ((static_cast<int64_t>(b) * a.K + z) * a.L + i) * a.V * esz;
}

// last request whose first window row is <= r
__device__ __forceinline__ int request_of_row(const int* rowoff, int B, int64_t r) {
  int lo = 0, hi = B - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (rowoff[mid] <= r) lo = mid; else hi = mid - 1;
  }
  return lo;
}

template <int DT>
__global__ void __launch_bounds__(kFT, 1) k_verify_fused(FusedArgs a) {
  constexpr int E = Elem<DT>::kPerVec;
  constexpr int ES = Elem<DT>::kBytes;
  extern __shared__ __align__(128) unsigned char smem[];
  unsigned char* stages = smem;
  FusedShared& sh = *reinterpret_cast<FusedShared*>(smem + kFusedStages * kFusedStageBytes);
  int* rowoff = reinterpret_cast<int*>(&sh + 1);  // [B + 1] window row offset of each request
  int* toff = rowoff + a.B + 1;                    // [B] target row of (b, 0)
  unsigned long long* mine = reinterpret_cast<unsigned long long*>(toff + a.B + 1);  // [B] units of request b streamed here (8-byte aligned: 2B + 2 ints precede)

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int B = a.B, K = a.K;
  const int G = gridDim.x, cta = blockIdx.x;
  pdl_wait();
  const uint64_t deadline = gtime() + kWaitNs;

  // ---- setup: request lengths -> window row offsets; this block's units
  for (int b = tid; b < B; b += kFT) {
    int l = a.vlen ? a.vlen[b] : a.L;
    if (l < 0 || l > a.L) l = 0;  // flagged where the request is decided
    rowoff[b] = (K + 1) * l;
    toff[b] = a.row_off ? a.row_off[b] : b * (a.L + 1);
    mine[b] = 0;
  }
  __syncthreads();
  const int total_rows = block_exclusive_scan<kFT>(rowoff, B, sh.scan_tmp);
  if (tid == 0) {
    rowoff[B] = total_rows;
    sh.epoch = __ldcg(a.ctl);
    sh.abort_ = 0;
    sh.flags = 0;
    for (int s = 0; s < kFusedStages; ++s) {
      mbar_init(&sh.full[s], 1);
      mbar_init(&sh.empty[s], kCW);
    }
    mbar_init(&sh.dbar, kCW);
    mbar_init(&sh.ddone, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  pdl_trigger();
  const int epoch = sh.epoch;
  volatile int* abort_flag = &sh.abort_;
  const int64_t Vu = a.Vu;
  const int64_t N = static_cast<int64_t>(total_rows) * Vu;
  const int64_t e_lo = split_start(cta, N, G), e_hi = split_start(cta + 1, N, G);
  const int64_t r_first = e_lo / Vu;
  if (tid < 64 && e_hi > e_lo && r_first + tid <= (e_hi - 1) / Vu) {
    const int64_t r = r_first + tid;
    const int b = request_of_row(rowoff, B, r);
    const int q = static_cast<int>(r - rowoff[b]);
    const int ell = (rowoff[b + 1] - rowoff[b]) / (K + 1);
    sh.rtok[tid] = __ldg(a.tokens + static_cast<int64_t>(b) * a.L + (q < ell ? q : (q - ell) % ell));
  }
  __syncthreads();

  if (warp == kCW) {
    // ================================================================ producer
    if (lane == 0) {
      int s = 0;
      uint32_t round = 0;
      int filled[kFusedStages];  // round in which each stage was last armed, -1 if never
#pragma unroll
      for (int t = 0; t < kFusedStages; ++t) filled[t] = -1;
      auto next_stage = [&]() -> StageMeta* {
        if (!mbar_wait(&sh.empty[s], (round & 1) ^ 1, deadline)) {
          atomicOr(a.status, kFlagTimeout);
          *abort_flag = 1;
          return nullptr;
        }
        filled[s] = static_cast<int>(round);
        return &sh.meta[s];
      };
      auto advance = [&]() {
        if (++s == kFusedStages) {
          s = 0;
          ++round;
        }
      };
      // ---- phase 1: this block's share of the window, chunk by chunk
      for (int64_t e = e_lo; e < e_hi && !*abort_flag;) {
        const int64_t r = e / Vu;
        const int64_t seg_hi = min(e_hi, (r + 1) * Vu);
        const int b = request_of_row(rowoff, B, r);
        const int q = static_cast<int>(r - rowoff[b]);
        const int ell = (rowoff[b + 1] - rowoff[b]) / (K + 1);
        const char* rowp = window_row<DT>(a, toff, b, ell, q);
        const int pos = q < ell ? q : (q - ell) % ell;
        int x = -1;
        bool have_x = r - r_first < 64;
        if (have_x) x = sh.rtok[r - r_first];
        for (int64_t u = e; u < seg_hi; u += kFusedStageBytes / 16) {
          const int n = static_cast<int>(seg_hi - u < kFusedStageBytes / 16 ? seg_hi - u : kFusedStageBytes / 16);
          StageMeta* mt = next_stage();
          if (!mt) break;
          const int64_t cu = u - r * Vu;  // first unit of the chunk inside the row
          mbar_expect_tx(&sh.full[s], static_cast<uint32_t>(n) * 16u);
          bulk_load(stages + s * kFusedStageBytes, rowp + cu * 16, static_cast<uint32_t>(n) * 16u, &sh.full[s]);
          if (!have_x) {  // the drafted token of this row, loaded while the first copy flies
            x = __ldg(a.tokens + static_cast<int64_t>(b) * a.L + pos);
            have_x = true;
          }
          const int64_t t = static_cast<int64_t>(x) - cu * E;
          mt->kind = kItemStats;
          mt->b = b;
          mt->n = n;
          mt->row = static_cast<int>(r);
          mt->slot = cta + static_cast<int>(r);
          mt->tok = (x >= 0 && x < a.V && t >= 0 && t < static_cast<int64_t>(n) * E) ? static_cast<int>(t) : -1;
          mt->seg_end = u + n == seg_hi;
          mt->seg_units = static_cast<int>(seg_hi - e);
          mbar_arrive(&sh.full[s]);
          advance();
        }
        e = seg_hi;
      }
      if (StageMeta* mt = *abort_flag ? nullptr : next_stage()) {
        mt->kind = kItemPhaseEnd;
        mbar_arrive(&sh.full[s]);
        advance();
      }
      // ---- phase 2: terminal chunks t = cta, cta + G, ... of the B * Pt
      for (int t = cta; t < B * a.Pt && !*abort_flag; t += G) {
        const int b = t / a.Pt, p = t - b * a.Pt;
        const int ell = (rowoff[b + 1] - rowoff[b]) / (K + 1);
        int j = 0, flags = 0;
        if (ell == 0) {
          const bool bad_len = a.vlen && (a.vlen[b] < 0 || a.vlen[b] > a.L);
          flags = bad_len ? kFlagVerifyLen : 0;  // nothing to test: a bonus draw from row 0
        } else {
          while (ld_acquire(a.dready + b) != epoch + 1) {
            if (gtime() > deadline) {
              atomicOr(a.status, kFlagTimeout);
              *abort_flag = 1;
              break;
            }
            __nanosleep(128);
          }
          if (*abort_flag) break;
          j = __ldcg(&a.dec[b].j);
          flags = __ldcg(&a.dec[b].flags);
        }
        StageMeta* mt = next_stage();
        if (!mt) break;
        mt->b = b;
        mt->slot = p;
        mt->j = j;
        mt->flags = flags;
        mt->ell = ell;
        if (flags) {
          mt->kind = kItemTermNoop;
        } else {
          const int64_t g0 = p * a.Vq / a.Pt, g1 = (p + 1) * a.Vq / a.Pt;
          const int n = static_cast<int>((g1 - g0) * 8);
          const int64_t v0 = g0 * 8;
          const bool resid = j < ell;
          const uint32_t seg = static_cast<uint32_t>(n) * ES;
          mbar_expect_tx(&sh.full[s], seg * (resid ? K + 1 : 1) + static_cast<uint32_t>(n) * 4u);
          unsigned char* buf = stages + s * kFusedStageBytes;
          bulk_load(buf, static_cast<const char*>(a.target) + ((static_cast<int64_t>(toff[b]) + j) * a.V + v0) * ES,
                    seg, &sh.full[s]);
          if (resid)
            for (int z = 0; z < K; ++z)
              bulk_load(buf + seg * (1 + z),
                        static_cast<const char*>(a.draft) +
                            (((static_cast<int64_t>(b) * K + z) * a.L + j) * a.V + v0) * ES,
                        seg, &sh.full[s]);
          bulk_load(buf + seg * (K + 1), a.g + (static_cast<int64_t>(b) * (a.L + 1) + j) * a.V + v0,
                    static_cast<uint32_t>(n) * 4u, &sh.full[s]);
          mt->kind = kItemTerm;
          mt->n = n;
          mt->v0 = static_cast<int>(v0);
          if (resid) {
            mt->ct = __ldcg(&a.dec[b].ct);
            mt->mt = __ldcg(&a.dec[b].mt);
            for (int z = 0; z < K; ++z) {
              mt->cz[z] = __ldcg(&a.dec[b].cz[z]);
              mt->mz[z] = __ldcg(&a.dec[b].mz[z]);
            }
          }
        }
        mbar_arrive(&sh.full[s]);
        advance();
      }
      if (StageMeta* mt = next_stage()) {
        mt->kind = kItemEnd;
        mbar_arrive(&sh.full[s]);
        advance();
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
    // Warps work independently: no block-wide barrier in the stream. Each warp
    // keeps per-thread statistics of the current row segment, writes its own
    // partial (row, block, warp) where the segment ends, and adds the units it
    // covered to the request's counter (release) when it moves to another
    // request. The only cross-warp step is inside a decision, synchronised by
    // bounded mbarrier waits.
    const int ctid = tid;
    int s = 0;
    uint32_t round = 0, dround = 0;
    float m = -INFINITY, sum = 0.f;
    int cur_b = -1;
    unsigned long long cur_units = 0;
    auto flush_units = [&]() {
      if (cur_b >= 0 && cur_units) {
        __threadfence();  // this warp's partials and token logits before its count
        __syncwarp();
        if (lane == 0) atomicAdd(a.req_units + cur_b, cur_units);
      }
      cur_units = 0;
    };
    for (;;) {
      if (!mbar_wait(&sh.full[s], round & 1, deadline)) {
        atomicOr(a.status, kFlagTimeout);
        *abort_flag = 1;
      }
      if (*abort_flag) break;
      const StageMeta& mt = sh.meta[s];
      const int kind = mt.kind;
      if (kind == kItemEnd) break;
      const unsigned char* buf = stages + s * kFusedStageBytes;
      if (kind == kItemStats) {
        const uint4* sv = reinterpret_cast<const uint4*>(buf);
        const int n = mt.n, tok = mt.tok, row = mt.row, slot = mt.slot, seg_end = mt.seg_end, b = mt.b;
        const int seg_units = mt.seg_units;
        if (ctid + 3 * kCT < n) {
          const uint4 v[4] = {sv[ctid], sv[ctid + kCT], sv[ctid + 2 * kCT], sv[ctid + 3 * kCT]};
          fold_vectors<DT, 4>(v, m, sum, a.k);
        } else {
          for (int u = ctid; u < n; u += kCT) {
            const uint4 v[1] = {sv[u]};
            fold_vectors<DT, 1>(v, m, sum, a.k);
          }
        }
        if (tok >= 0 && (tok / E) % kCT == ctid) {
          float xv[E];
          Elem<DT>::unpack(sv[tok / E], xv);
          a.xg[row] = xv[tok % E];
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.empty[s]);
        if (seg_end) {
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) {
            const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
            const float s2 = __shfl_xor_sync(0xffffffffu, sum, o);
            ms_merge(m, sum, m2, s2, a.k);
          }
          if (lane == 0) a.part[static_cast<int64_t>(slot) * kCW + warp] = make_float2(m, sum);
          m = -INFINITY;
          sum = 0.f;
          if (b != cur_b) {
            flush_units();
            cur_b = b;
          }
          cur_units += static_cast<unsigned long long>(seg_units);
        }
      } else if (kind == kItemPhaseEnd) {
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.empty[s]);
        flush_units();
        // ---- the decisions this block owns: request db is decided by the
        // block holding its last window unit
        const int b_first = e_hi > e_lo ? request_of_row(rowoff, B, e_lo / Vu) : B;
        const int b_last = e_hi > e_lo ? request_of_row(rowoff, B, (e_hi - 1) / Vu) : -1;
        for (int db = b_first; db <= b_last; ++db) {
          const int base = rowoff[db], nrows = rowoff[db + 1] - rowoff[db];
          if (nrows == 0) continue;
          const int64_t last_unit = static_cast<int64_t>(base + nrows) * Vu - 1;
          if (last_unit < e_lo || last_unit >= e_hi) continue;
          // every warp of every block streaming db has counted its units
          if (lane == 0) {
            const unsigned long long want =
                static_cast<unsigned long long>(nrows) * static_cast<unsigned long long>(Vu) * kCW;
            while (ld_acquire_u64(a.req_units + db) != want) {
              if (gtime() > deadline) {
                atomicOr(a.status, kFlagTimeout);
                *abort_flag = 1;
                break;
              }
              __nanosleep(64);
            }
          }
          __syncwarp();
          if (*abort_flag) break;
          const int ell = nrows / (K + 1);
          if (warp == 0) {
            if (lane < ell) {
              const int x = __ldg(a.tokens + static_cast<int64_t>(db) * a.L + lane);
              if (x < 0 || x >= a.V) atomicOr(&sh.flags, kFlagTokenRange);
              sh.d_x[lane] = x;
            }
          }
          // rows q = warp, warp + 16, ...: merge the (piece, warp) partials across the lanes
          for (int q = warp; q < nrows; q += kCW) {
            const int64_t r = base + q;
            const int64_t c0 = owner_of(r * Vu, N, G), c1 = owner_of((r + 1) * Vu - 1, N, G);
            const int np = static_cast<int>(c1 - c0 + 1) * kCW;
            float mm = -INFINITY, ss = 0.f;
            for (int t = lane; t < np; t += 64) {
              float2 pr[2];
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                const int tt = t + 32 * h;
                const int64_t c = c0 + tt / kCW;
                pr[h] = tt < np && (N >= G || split_start(c + 1, N, G) > split_start(c, N, G))
                            ? __ldcg(a.part + (c + r) * kCW + tt % kCW)
                            : make_float2(-INFINITY, 0.f);
              }
              ms_merge(mm, ss, pr[0].x, pr[0].y, a.k);
              ms_merge(mm, ss, pr[1].x, pr[1].y, a.k);
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
              const float m2 = __shfl_xor_sync(0xffffffffu, mm, o);
              const float s2 = __shfl_xor_sync(0xffffffffu, ss, o);
              ms_merge(mm, ss, m2, s2, a.k);
            }
            if (lane == 0) {
              sh.d_m[q] = mm;
              sh.d_s[q] = ss;
              sh.d_xg[q] = __ldcg(a.xg + r);
              if (!isfinite(mm) || !isfinite(ss)) atomicOr(&sh.flags, kFlagNonFinite);
            }
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(&sh.dbar);
          if (warp == 0) {
            if (!mbar_wait(&sh.dbar, dround & 1, deadline)) {
              atomicOr(a.status, kFlagTimeout);
              *abort_flag = 1;
            }
            int flags = sh.flags;
            __syncwarp();
            if (lane == 0) sh.flags = 0;  // for the next decision: no warp writes it before ddone
            DecideOut o = {};
            o.j = -1;
            if (!flags && !*abort_flag) {
              const DecideIn in{sh.d_xg, sh.d_m, sh.d_s, sh.d_x, ell, K, a.L, a.T};
              o = decide_warp(in, a.u + static_cast<int64_t>(db) * a.L,
                              a.mix_w ? a.mix_w + static_cast<int64_t>(db) * K : nullptr);
              if (o.bad) flags |= kFlagNonFinite;
            }
            if (lane == 0) {
              Decision& d = a.dec[db];
              d.j = o.j;
              d.flags = flags;
              d.ell = ell;
              d.ct = o.ct;
              d.mt = o.mt;
              for (int z = 0; z < kMaxK; ++z) {
                d.cz[z] = z < K ? o.cz[z] : 0.f;
                d.mz[z] = z < K ? o.mz[z] : 0.f;
              }
              a.req_units[db] = 0ull;
              __threadfence();
              st_release(a.dready + db, epoch + 1);
              mbar_arrive(&sh.ddone);
            }
          }
          // the shared row buffers are reused by the next decision of this block
          if (!mbar_wait(&sh.ddone, dround & 1, deadline)) {
            atomicOr(a.status, kFlagTimeout);
            *abort_flag = 1;
          }
          ++dround;
          if (*abort_flag) break;
        }
      } else {
        // ---- terminal chunk: best residual and bonus scores over [v0, v0 + n);
        // every warp publishes its maxima (the last block out reads them)
        Best br{-INFINITY, -1}, bb{-INFINITY, -1};
        const int b = mt.b, j = mt.j, ell = mt.ell;
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
        if (lane == 0 && kind == kItemTerm) {
          if (br.idx >= 0) red_max_u64(a.keys + 2 * b, score_key(br.score, br.idx));
          if (bb.idx >= 0) red_max_u64(a.keys + 2 * b + 1, score_key(bb.score, bb.idx));
        }
      }
      if (++s == kFusedStages) {
        s = 0;
        ++round;
      }
    }
  }

  // ---- exit: the last block out writes every request's outputs, clears the
  // keys and advances the epoch
  __threadfence();  // every thread's key maxima before the exit count
  __syncthreads();
  if (tid == 0) {
    sh.last = atomicAdd(a.ctl + 2, 1) == G - 1;
  }
  __syncthreads();
  if (!sh.last) return;
  __threadfence();
  for (int t = tid; t < B * (a.L + 1); t += kFT) {
    const int b = t / (a.L + 1), i = t - b * (a.L + 1);
    const int ell = (rowoff[b + 1] - rowoff[b]) / (K + 1);
    int j = 0, flags = 0;
    if (ell == 0) {
      flags = a.vlen && (a.vlen[b] < 0 || a.vlen[b] > a.L) ? kFlagVerifyLen : 0;
    } else {
      j = __ldcg(&a.dec[b].j);
      flags = __ldcg(&a.dec[b].flags);
    }
    if (*abort_flag) flags |= kFlagTimeout;
    const unsigned long long kr = __ldcg(a.keys + 2 * b), kb = __ldcg(a.keys + 2 * b + 1);
    const int tk = i < j ? __ldg(a.tokens + static_cast<int64_t>(b) * a.L + i) : -1;
    const int term = flags ? -1 : ((j < ell && kr) ? key_token(kr) : key_token(kb));
    const bool ok = flags == 0 && term >= 0;
    a.out_tokens[static_cast<int64_t>(b) * (a.L + 1) + i] = !ok ? -1 : (i < j ? tk : (i == j ? term : -1));
    if (i == 0) {
      a.accept_len[b] = ok ? j : -1;
      if (flags) atomicOr(a.status, flags);
      else if (!ok) atomicOr(a.status, kFlagNonFinite);
    }
  }
  __syncthreads();  // every output thread has read the keys before they are cleared
  for (int t = tid; t < 2 * B; t += kFT) a.keys[t] = 0ull;
  if (tid == 0) {
    a.ctl[2] = 0;
    __threadfence();
    a.ctl[0] = epoch + 1;
  }
}

// ------------------------------------------------------------------- host

int fused_pt(int64_t V, int dtype, int K) {
  const int64_t es = dtype == 0 ? 4 : 2;
  const int64_t per_group = 8 * (es * (K + 1) + 4);  // bytes of 8 elements of every operand
  const int64_t groups = kFusedStageBytes / per_group;
  const int64_t Vq = V / 8;
  return static_cast<int>(std::max<int64_t>(1, (Vq + groups - 1) / groups));
}

size_t fused_smem_bytes(int B) {
  return static_cast<size_t>(kFusedStages) * kFusedStageBytes + sizeof(FusedShared) +
         static_cast<size_t>(2 * B + 2) * sizeof(int) + static_cast<size_t>(B) * sizeof(unsigned long long);
}

cudaError_t launch_fused(const FusedArgs& a, int dtype, int grid, cudaStream_t st) {
  const size_t smem = fused_smem_bytes(a.B);
  void (*kern)(FusedArgs) = dtype == 0 ? k_verify_fused<0> : k_verify_fused<1>;
  const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, dim3(grid), dim3(kFT), smem, st, a);
}

}  // namespace specv
