// C ABI of specv (declared in include/specv.h): host-side argument checks,
// workspace carving and kernel launches. No call allocates, frees or
// synchronises; every launch is stream-ordered.
#include <algorithm>
#include <cmath>
#include <mutex>

#include <cuda.h>  // driver API types only (no driver functions are linked)

#include "specv.h"
#include "common.cuh"
#include "internal.h"

using namespace specv;

namespace {

constexpr size_t kHeader = 256;  // status word + padding

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }
bool aligned(const void* p, size_t a) { return reinterpret_cast<uintptr_t>(p) % a == 0; }  // NULL is aligned
int esize(int dtype) { return dtype == SPEC_F32 ? 4 : 2; }
bool dtype_ok(int dtype) { return dtype == SPEC_F32 || dtype == SPEC_BF16; }

int map_cuda(cudaError_t e) { return e == cudaSuccess ? SPEC_OK : SPEC_ERR_CUDA; }

int sm_count() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  static std::mutex mu;
  static int cache[64] = {0};
  std::lock_guard<std::mutex> lock(mu);
  if (dev < 64 && cache[dev]) return cache[dev];
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1) sms = 148;
  if (dev < 64) cache[dev] = sms;
  return sms;
}

// Fixed scratch of spec_softmax_T_noalloc: the per-row statistics partials of
// at most SPEC_NOALLOC_MAX_ROWS rows (kGMax + rows slots, as in the softmax
// workspace after its header). Shared by every call on a device.
static __device__ __align__(256) float2 g_noalloc_part[kGMax + SPEC_NOALLOC_MAX_ROWS];

// Id of the current CUDA context, unique over the life of the process (0 if
// there is none yet or the driver cannot say). The two driver functions are
// fetched through the runtime, so the library does not link the driver.
unsigned long long current_context_id() {
  using GetCurrent = CUresult (*)(CUcontext*);
  using GetId = CUresult (*)(CUcontext, unsigned long long*);
  static GetCurrent get_current = nullptr;
  static GetId get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &f, 4000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<GetCurrent>(f);
    f = nullptr;
    q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &f, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<GetId>(f);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Device address of g_noalloc_part in the current context: looked up with
// cudaGetSymbolAddress once per context (a device's primary context, with
// that device current) and cached under the context's id. A device reset
// ends the context, and the next call looks the address up again in the new
// one. If the context id is unavailable the address is looked up every call.
int noalloc_scratch(float2** out) {
  struct Entry {
    unsigned long long ctx;
    void* ptr;
  };
  static std::mutex mu;
  static Entry cache[64] = {};
  static int next = 0;
  const unsigned long long id = current_context_id();
  if (id) {
    std::lock_guard<std::mutex> lock(mu);
    for (const Entry& e : cache)
      if (e.ctx == id) {
        *out = static_cast<float2*>(e.ptr);
        return SPEC_OK;
      }
  }
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_part) != cudaSuccess || !p) return SPEC_ERR_CUDA;
  const unsigned long long id2 = id ? id : current_context_id();  // the lookup may have created the context
  if (id2) {
    std::lock_guard<std::mutex> lock(mu);
    cache[next] = Entry{id2, p};
    next = (next + 1) % 64;
  }
  *out = static_cast<float2*>(p);
  return SPEC_OK;
}

// Resident sampling blocks per SM (cached per device and kernel variant).
int accept_slots(int dtype, bool vec, int K, bool topp) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 1;
  static std::mutex mu;
  static int cache[64][16] = {};
  std::lock_guard<std::mutex> lock(mu);
  int& c = cache[dev][(topp ? 8 : 0) + dtype * 4 + (vec ? 2 : 0) + (K == 1 ? 1 : 0)];
  if (!c) c = accept_blocks_per_sm(dtype, vec, K, topp);
  return c;
}

// Verify workspace: persistent state first (zero between calls), then scratch.
// The walk has B (K+1) L rows, plus one bonus row per request with top-p
// filtering, whose nucleus kernels add five per-row arrays.
struct VerifyLayout {
  size_t ticket, keys;     // persistent: per-request tickets [B], terminal keys [2B]
  size_t xg, rpart;        // scratch
  size_t nm, nlf, nkey, nv;  // top-p scratch: row maxima, log nucleus masses, cut keys, cut tokens,
  size_t nflag;              // and the rows the fast nucleus kernel hands to the exact one
  size_t total;
};

size_t walk_rows(int B, int L, int K, bool topp) {
  return static_cast<size_t>(B) * (static_cast<size_t>(K + 1) * L + (topp ? 1 : 0));
}

VerifyLayout verify_layout(int B, int L, int K, int64_t V, bool topp = false) {
  (void)V;
  VerifyLayout l;
  const size_t rows = walk_rows(B, L, K, topp);
  l.ticket = kHeader;
  l.keys = l.ticket + align256(static_cast<size_t>(B) * sizeof(int));
  l.xg = l.keys + align256(static_cast<size_t>(2 * B) * sizeof(unsigned long long));
  l.rpart = l.xg + align256(rows * sizeof(float));
  l.total = l.rpart + align256((static_cast<size_t>(kGMax) + rows) * sizeof(float2));
  l.nm = l.nlf = l.nkey = l.nv = l.nflag = 0;
  if (topp) {
    l.nm = l.total;
    l.nlf = l.nm + align256(rows * sizeof(float));
    l.nkey = l.nlf + align256(rows * sizeof(double));
    l.nv = l.nkey + align256(rows * sizeof(uint32_t));
    l.nflag = l.nv + align256(rows * sizeof(int32_t));
    l.total = l.nflag + align256(rows * sizeof(int));
  }
  return l;
}

bool verify_shape_ok(int B, int L, int K) {
  return B >= 1 && B <= SPEC_MAX_B && L >= 0 && L <= SPEC_MAX_L && K >= 1 && K <= SPEC_MAX_K;
}

// Checks shared by the verify entry points. Returns SPEC_OK or a negative status.
int verify_check(const void* target, const int32_t* row_off, const void* draft, const float* mix_w, int K,
                 int dtype, const int32_t* tokens, const int32_t* vlen, const float* u, const float* g, int B, int L,
                 int64_t V, float T, const int32_t* accept_len, const int32_t* out_tokens, const void* ws,
                 size_t ws_bytes, bool accept_stage, bool topp = false) {
  // [B, L] and [B, K, L, V] arrays are empty when L == 0, so their pointers may then be NULL.
  if (!target || (L > 0 && !draft)) return SPEC_ERR_ARG;
  if (accept_stage && (!g || !accept_len || !out_tokens || (L > 0 && (!tokens || !u)))) return SPEC_ERR_ARG;
  if (!dtype_ok(dtype) || V < 1 || !(T > 0.f) || !std::isfinite(T)) return SPEC_ERR_ARG;
  if (B < 1 || L < 0 || K < 1) return SPEC_ERR_ARG;
  if (!verify_shape_ok(B, L, K) || V > SPEC_MAX_V) return SPEC_ERR_UNSUPPORTED;
  if (accept_stage && K > 1 && !mix_w) return SPEC_ERR_ARG;
  if (!ws) return SPEC_ERR_WORKSPACE;
  if (ws_bytes < verify_layout(B, L, K, V, topp).total) return SPEC_ERR_WORKSPACE;
  const int es = esize(dtype);
  if (!aligned(target, es) || !aligned(draft, es) || !aligned(g, 4) || !aligned(u, 4) || !aligned(tokens, 4) ||
      !aligned(accept_len, 4) || !aligned(out_tokens, 4) || !aligned(ws, 16) || !aligned(row_off, 4) ||
      !aligned(vlen, 4) || !aligned(mix_w, 4))
    return SPEC_ERR_ARG;
  return SPEC_OK;
}

// The statistics stage's vector decision; the accept stage must use the same
// units per row and grid to find the partials.
bool stats_vec(const void* target, const void* draft, int dtype, int64_t V) {
  return (V * esize(dtype)) % 16 == 0 && aligned(target, 16) && aligned(draft, 16);
}

// The walk of the statistics stage (bonus rows with top-p filtering).
RowSpace verify_walk(const void* target, const int32_t* row_off, const void* draft, int K, const int32_t* tokens,
                     const int32_t* vlen, int B, int L, int64_t V, float* xg, bool topp) {
  RowSpace rs = {};
  rs.target = target;
  rs.draft = draft;
  rs.row_off = row_off;
  rs.vlen = vlen;
  rs.tokens = tokens;
  rs.xg = xg;
  rs.stride = V;
  rs.rows = 0;
  rs.B = B;
  rs.L = L;
  rs.K = K;
  rs.verify = 1;
  rs.bonus = topp ? 1 : 0;
  return rs;
}

int stats_grid_of(int dtype, bool vec, int B, int L, int K, int64_t V, bool topp) {
  const int64_t Vu = units_per_row(V, dtype, vec);
  return stats_grid(dtype, vec, static_cast<int64_t>(walk_rows(B, L, K, topp)) * Vu, Vu);
}

int launch_stats_stage(const void* target, const int32_t* row_off, const void* draft, int K, int dtype,
                       const int32_t* tokens, const int32_t* vlen, int B, int L, int64_t V, float T, void* ws,
                       cudaStream_t st, bool topp = false) {
  if (L == 0 && !topp) return SPEC_OK;
  const bool vec = stats_vec(target, draft, dtype, V);
  const VerifyLayout lay = verify_layout(B, L, K, V, topp);
  RowSpace rs = verify_walk(target, row_off, draft, K, tokens, vlen, B, L, V,
                            reinterpret_cast<float*>(static_cast<char*>(ws) + lay.xg), topp);
  const int G = stats_grid_of(dtype, vec, B, L, K, V, topp);
  return map_cuda(launch_row_stats(rs, dtype, vec, V, T, G, reinterpret_cast<float2*>(static_cast<char*>(ws) + lay.rpart), st));
}

int launch_nucleus_stage(const void* target, const int32_t* row_off, const void* draft, int K, int dtype,
                         const int32_t* tokens, const int32_t* vlen, int B, int L, int64_t V, float T, float top_p,
                         void* ws, cudaStream_t st) {
  const bool vec = stats_vec(target, draft, dtype, V);
  const VerifyLayout lay = verify_layout(B, L, K, V, true);
  char* w = static_cast<char*>(ws);
  NucleusArgs a = {};
  a.rs = verify_walk(target, row_off, draft, K, tokens, vlen, B, L, V, reinterpret_cast<float*>(w + lay.xg), true);
  a.V = V;
  a.k = static_cast<float>(1.4426950408889634 / static_cast<double>(T));
  a.top_p = static_cast<double>(top_p);
  a.row_m = reinterpret_cast<float*>(w + lay.nm);
  a.row_lf = reinterpret_cast<double*>(w + lay.nlf);
  a.cut_key = reinterpret_cast<uint32_t*>(w + lay.nkey);
  a.cut_v = reinterpret_cast<int32_t*>(w + lay.nv);
  // bf16 rows of 16-byte vectors: the windowed kernel first, the exact one for the rows it hands over
  if (dtype == 1 && vec && V >= kNucFastMinV) {
    a.flags = reinterpret_cast<int*>(w + lay.nflag);
    const cudaError_t e = launch_nucleus_fast(a, st);
    if (e != cudaSuccess) return map_cuda(e);
    a.only = a.flags;
  }
  return map_cuda(launch_nucleus(a, dtype, vec, st));
}

int launch_accept_stage(const void* target, const int32_t* row_off, const void* draft, const float* mix_w, int K,
                        int dtype, const int32_t* tokens, const int32_t* vlen, const float* u, const float* g, int B,
                        int L, int64_t V, float T, int32_t* accept_len, int32_t* out_tokens, void* ws,
                        cudaStream_t st, bool topp = false) {
  const bool vec = stats_vec(target, draft, dtype, V);
  const bool vec_term = vec && aligned(g, 16);
  const VerifyLayout lay = verify_layout(B, L, K, V, topp);
  char* w = static_cast<char*>(ws);
  VerifyArgs a = {};
  a.target = target;
  a.row_off = row_off;
  a.draft = draft;
  a.mix_w = mix_w;
  a.tokens = tokens;
  a.vlen = vlen;
  a.u = u;
  a.g = g;
  a.B = B;
  a.L = L;
  a.K = K;
  a.V = V;
  a.T = T;
  a.accept_len = accept_len;
  a.out_tokens = out_tokens;
  a.status = reinterpret_cast<int*>(w);
  a.tickets = reinterpret_cast<int*>(w + lay.ticket);
  a.keys = reinterpret_cast<unsigned long long*>(w + lay.keys);
  a.xg = reinterpret_cast<const float*>(w + lay.xg);
  a.rpart = reinterpret_cast<const float2*>(w + lay.rpart);
  a.Vu = units_per_row(V, dtype, vec);
  a.G = stats_grid_of(dtype, vec, B, L, K, V, topp);
  a.topp = topp ? 1 : 0;
  if (topp) {
    a.nuc_m = reinterpret_cast<const float*>(w + lay.nm);
    a.nuc_lf = reinterpret_cast<const double*>(w + lay.nlf);
    a.nuc_key = reinterpret_cast<const uint32_t*>(w + lay.nkey);
    a.nuc_v = reinterpret_cast<const int32_t*>(w + lay.nv);
  }
  // Blocks per request for the terminal row: the whole (P, B) grid resident
  // at once (no second wave), at least 256 units of the row per block.
  const int64_t term_units = vec_term ? V / (16 / esize(dtype)) : V;
  const int64_t slots = static_cast<int64_t>(sm_count()) * accept_slots(dtype, vec_term, K, topp);
  const int64_t p_fit = std::max<int64_t>(1, slots / B);
  a.P = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>({p_fit, kPMax, term_units / kThreads})));
  return map_cuda(launch_accept_sample(a, dtype, vec_term, st));
}

// top_p >= 1: unfiltered (two stages); below 1: the nucleus kernel (which
// also finds every row's maximum and the drafted-token logits, in place of
// the statistics stage) over the window with bonus rows, then the filtered
// accept / sample stage.
int verify_common(const void* target, const int32_t* row_off, const void* draft, const float* mix_w, int K,
                  int dtype, const int32_t* tokens, const int32_t* vlen, const float* u, const float* g, int B,
                  int L, int64_t V, float T, int32_t* accept_len, int32_t* out_tokens, void* ws, size_t ws_bytes,
                  cudaStream_t st, float top_p = 1.f) {
  if (!(top_p > 0.f && top_p <= 1.f)) return SPEC_ERR_ARG;  // NaN included
  const bool topp = top_p < 1.f;
  int e = verify_check(target, row_off, draft, mix_w, K, dtype, tokens, vlen, u, g, B, L, V, T, accept_len,
                       out_tokens, ws, ws_bytes, true, topp);
  if (e) return e;
  e = topp ? launch_nucleus_stage(target, row_off, draft, K, dtype, tokens, vlen, B, L, V, T, top_p, ws, st)
           : launch_stats_stage(target, row_off, draft, K, dtype, tokens, vlen, B, L, V, T, ws, st);
  if (e) return e;
  return launch_accept_stage(target, row_off, draft, mix_w, K, dtype, tokens, vlen, u, g, B, L, V, T, accept_len,
                             out_tokens, ws, st, topp);
}

}  // namespace

extern "C" {

const char* spec_status_string(int status) {
  switch (status) {
    case SPEC_OK: return "SPEC_OK";
    case SPEC_ERR_ARG: return "SPEC_ERR_ARG: invalid argument (null pointer, size, alignment, T or budget)";
    case SPEC_ERR_UNSUPPORTED: return "SPEC_ERR_UNSUPPORTED: shape outside the supported limits";
    case SPEC_ERR_CUDA: return "SPEC_ERR_CUDA: a kernel launch failed";
    case SPEC_ERR_WORKSPACE: return "SPEC_ERR_WORKSPACE: workspace missing or too small";
    default: return "unknown spec_status";
  }
}

size_t spec_softmax_workspace_size(int64_t rows) {
  if (rows < 0 || rows > (int64_t{1} << 31)) return 0;
  return kHeader + align256((static_cast<size_t>(kGMax) + static_cast<size_t>(rows)) * sizeof(float2));
}

size_t spec_verify_workspace_size(int B, int L, int K, int64_t V) {
  if (!verify_shape_ok(B, L, K) || V < 1 || V > SPEC_MAX_V) return 0;
  return verify_layout(B, L, K, V).total;
}

size_t spec_verify_top_p_workspace_size(int B, int L, int K, int64_t V) {
  if (!verify_shape_ok(B, L, K) || V < 1 || V > SPEC_MAX_V) return 0;
  return verify_layout(B, L, K, V, true).total;
}

size_t spec_dvl_workspace_size(int B) {
  if (B < 1 || B > SPEC_MAX_B) return 0;
  return 2 * kHeader;
}

int spec_workspace_init(void* workspace, size_t ws_bytes, spec_stream_t stream) {
  if (!workspace || ws_bytes == 0) return SPEC_ERR_ARG;
  return map_cuda(cudaMemsetAsync(workspace, 0, ws_bytes, reinterpret_cast<cudaStream_t>(stream)));
}

int spec_softmax_T(const void* logits, int dtype, int64_t rows, int64_t V, int64_t row_stride, float T,
                   float* row_max, float* row_lse, float* probs, void* workspace, size_t ws_bytes,
                   spec_stream_t stream) {
  if (!logits || !row_max || !row_lse) return SPEC_ERR_ARG;
  if (!dtype_ok(dtype) || rows < 0 || V < 1 || V > 0x7fffffffLL || row_stride < V || !(T > 0.f) ||
      !std::isfinite(T))
    return SPEC_ERR_ARG;
  if (rows > (int64_t{1} << 31)) return SPEC_ERR_UNSUPPORTED;
  if (!workspace) return SPEC_ERR_WORKSPACE;
  if (ws_bytes < spec_softmax_workspace_size(rows)) return SPEC_ERR_WORKSPACE;
  const int es = esize(dtype);
  if (!aligned(logits, es) || !aligned(row_max, 4) || !aligned(row_lse, 4) || (probs && !aligned(probs, 4)) ||
      !aligned(workspace, 16))
    return SPEC_ERR_ARG;
  if (rows == 0) return SPEC_OK;
  const bool vec = (V * es) % 16 == 0 && (row_stride * es) % 16 == 0 && aligned(logits, 16) &&
                   (!probs || aligned(probs, 16));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  float2* part = reinterpret_cast<float2*>(static_cast<char*>(workspace) + kHeader);
  const int64_t Vu = units_per_row(V, dtype, vec);
  const int G = stats_grid(dtype, vec, rows * Vu, Vu);
  RowSpace rs = {};
  rs.target = logits;
  rs.stride = row_stride;
  rs.rows = rows;
  rs.verify = 0;
  int e = map_cuda(launch_row_stats(rs, dtype, vec, V, T, G, part, st));
  if (e) return e;
  return map_cuda(
      launch_softmax_finalize(logits, dtype, vec, rows, V, row_stride, T, G, part, row_max, row_lse, probs, st));
}

int spec_softmax_T_noalloc(const void* logits, int dtype, int64_t rows, int64_t V, int64_t row_stride, float T,
                           float* row_max, float* row_lse, float* probs, spec_stream_t stream) {
  if (!logits || !row_max || !row_lse) return SPEC_ERR_ARG;
  if (!dtype_ok(dtype) || rows < 0 || V < 1 || V > 0x7fffffffLL || row_stride < V || !(T > 0.f) ||
      !std::isfinite(T))
    return SPEC_ERR_ARG;
  if (rows > SPEC_NOALLOC_MAX_ROWS) return SPEC_ERR_UNSUPPORTED;  // beyond the fixed scratch
  const int es = esize(dtype);
  if (!aligned(logits, es) || !aligned(row_max, 4) || !aligned(row_lse, 4) || (probs && !aligned(probs, 4)))
    return SPEC_ERR_ARG;
  if (rows == 0) return SPEC_OK;
  float2* part = nullptr;
  const int se = noalloc_scratch(&part);
  if (se) return se;
  const bool vec = (V * es) % 16 == 0 && (row_stride * es) % 16 == 0 && aligned(logits, 16) &&
                   (!probs || aligned(probs, 16));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int64_t Vu = units_per_row(V, dtype, vec);
  const int G = stats_grid(dtype, vec, rows * Vu, Vu);
  RowSpace rs = {};
  rs.target = logits;
  rs.stride = row_stride;
  rs.rows = rows;
  rs.verify = 0;
  int e = map_cuda(launch_row_stats(rs, dtype, vec, V, T, G, part, st));
  if (e) return e;
  return map_cuda(
      launch_softmax_finalize(logits, dtype, vec, rows, V, row_stride, T, G, part, row_max, row_lse, probs, st));
}

int spec_verify_block(const void* target_logits, const int32_t* target_row_off, const void* draft_logits, int dtype,
                      const int32_t* draft_tokens, const int32_t* verify_len, const float* uniforms,
                      const float* gumbel, int B, int L, int64_t V, float T, int32_t* accept_len,
                      int32_t* out_tokens, void* workspace, size_t ws_bytes, spec_stream_t stream) {
  return verify_common(target_logits, target_row_off, draft_logits, nullptr, 1, dtype, draft_tokens, verify_len,
                       uniforms, gumbel, B, L, V, T, accept_len, out_tokens, workspace, ws_bytes,
                       reinterpret_cast<cudaStream_t>(stream));
}

int spec_verify_mixture(const void* target_logits, const int32_t* target_row_off, const void* draft_logits,
                        const float* mix_weights, int K, int dtype, const int32_t* draft_tokens,
                        const int32_t* verify_len, const float* uniforms, const float* gumbel, int B, int L,
                        int64_t V, float T, int32_t* accept_len, int32_t* out_tokens, void* workspace,
                        size_t ws_bytes, spec_stream_t stream) {
  if (!mix_weights) return SPEC_ERR_ARG;
  return verify_common(target_logits, target_row_off, draft_logits, mix_weights, K, dtype, draft_tokens, verify_len,
                       uniforms, gumbel, B, L, V, T, accept_len, out_tokens, workspace, ws_bytes,
                       reinterpret_cast<cudaStream_t>(stream));
}

int spec_verify_block_top_p(const void* target_logits, const int32_t* target_row_off, const void* draft_logits,
                            int dtype, const int32_t* draft_tokens, const int32_t* verify_len, const float* uniforms,
                            const float* gumbel, int B, int L, int64_t V, float T, float top_p,
                            int32_t* accept_len, int32_t* out_tokens, void* workspace, size_t ws_bytes,
                            spec_stream_t stream) {
  return verify_common(target_logits, target_row_off, draft_logits, nullptr, 1, dtype, draft_tokens, verify_len,
                       uniforms, gumbel, B, L, V, T, accept_len, out_tokens, workspace, ws_bytes,
                       reinterpret_cast<cudaStream_t>(stream), top_p);
}

int spec_verify_mixture_top_p(const void* target_logits, const int32_t* target_row_off, const void* draft_logits,
                              const float* mix_weights, int K, int dtype, const int32_t* draft_tokens,
                              const int32_t* verify_len, const float* uniforms, const float* gumbel, int B, int L,
                              int64_t V, float T, float top_p, int32_t* accept_len, int32_t* out_tokens,
                              void* workspace, size_t ws_bytes, spec_stream_t stream) {
  if (!mix_weights) return SPEC_ERR_ARG;
  return verify_common(target_logits, target_row_off, draft_logits, mix_weights, K, dtype, draft_tokens, verify_len,
                       uniforms, gumbel, B, L, V, T, accept_len, out_tokens, workspace, ws_bytes,
                       reinterpret_cast<cudaStream_t>(stream), top_p);
}

int spec_verify_window_stats(const void* target_logits, const int32_t* target_row_off, const void* draft_logits,
                             int K, int dtype, const int32_t* draft_tokens, const int32_t* verify_len, int B, int L,
                             int64_t V, float T, void* workspace, size_t ws_bytes, spec_stream_t stream) {
  if (L > 0 && !draft_tokens) return SPEC_ERR_ARG;
  const int e = verify_check(target_logits, target_row_off, draft_logits, nullptr, K, dtype, draft_tokens, verify_len,
                             nullptr, nullptr, B, L, V, T, nullptr, nullptr, workspace, ws_bytes, false);
  if (e) return e;
  return launch_stats_stage(target_logits, target_row_off, draft_logits, K, dtype, draft_tokens, verify_len, B, L, V, T,
                            workspace, reinterpret_cast<cudaStream_t>(stream));
}

int spec_verify_accept(const void* target_logits, const int32_t* target_row_off, const void* draft_logits,
                       const float* mix_weights, int K, int dtype, const int32_t* draft_tokens,
                       const int32_t* verify_len, const float* uniforms, const float* gumbel, int B, int L, int64_t V,
                       float T, int32_t* accept_len, int32_t* out_tokens, void* workspace, size_t ws_bytes,
                       spec_stream_t stream) {
  const int e = verify_check(target_logits, target_row_off, draft_logits, mix_weights, K, dtype, draft_tokens,
                             verify_len, uniforms, gumbel, B, L, V, T, accept_len, out_tokens, workspace, ws_bytes,
                             true);
  if (e) return e;
  return launch_accept_stage(target_logits, target_row_off, draft_logits, mix_weights, K, dtype, draft_tokens,
                             verify_len, uniforms, gumbel, B, L, V, T, accept_len, out_tokens, workspace,
                             reinterpret_cast<cudaStream_t>(stream));
}

int dvl_allocate_pack(const float* scores, int B, int L, int budget, int32_t* verify_len, int32_t* offsets,
                      int32_t* slot_map, const void* dense_target, void* packed_target, int dtype, int64_t V,
                      void* workspace, size_t ws_bytes, spec_stream_t stream) {
  if (B < 1 || L < 0 || budget < B) return SPEC_ERR_ARG;
  if ((!scores && L > 0) || !verify_len || !offsets) return SPEC_ERR_ARG;  // [B, 0] scores may be NULL
  if (B > SPEC_MAX_B || L > SPEC_MAX_L || static_cast<int64_t>(B) * L > SPEC_MAX_DVL_ELEMS)
    return SPEC_ERR_UNSUPPORTED;
  const bool pack = dense_target || packed_target;
  if (pack && (!dense_target || !packed_target || !dtype_ok(dtype) || V < 1 || V > 0x7fffffffLL))
    return SPEC_ERR_ARG;
  if (!aligned(scores, 4) || !aligned(verify_len, 4) || !aligned(offsets, 4) || (slot_map && !aligned(slot_map, 4)))
    return SPEC_ERR_ARG;
  if (pack && (!aligned(dense_target, esize(dtype)) || !aligned(packed_target, esize(dtype)))) return SPEC_ERR_ARG;
  if (!workspace) return SPEC_ERR_WORKSPACE;
  if (ws_bytes < spec_dvl_workspace_size(B) || !aligned(workspace, 16)) return SPEC_ERR_WORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int* status = static_cast<int*>(workspace);
  int e = map_cuda(launch_dvl(scores, B, L, budget, verify_len, offsets, slot_map, status, st));
  if (e || !pack) return e;
  return map_cuda(launch_pack(dense_target, packed_target, dtype, B, L, V, budget, offsets, st));
}

}  // extern "C"
