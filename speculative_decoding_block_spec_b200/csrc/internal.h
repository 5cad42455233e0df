// Host-side interfaces between the C-ABI layer (api.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace specv {

// The rows walked by the row-statistics kernel.
//  plain  (verify == 0): row r at target + r * stride elements, r < rows.
//  verify (verify == 1): request b contributes (K+1) * l_b + bonus rows, l_b =
//    verify_len[b] (L if NULL): first target rows 0..l_b-1, and row l_b too
//    when bonus == 1 (row of (b, i) is row_off[b] + i, or b*(L+1) + i when
//    row_off is NULL), then draft rows (z, i) for z < K, i < l_b at
//    draft + ((b*K + z)*L + i) * V.
struct RowSpace {
  const void* target;
  const void* draft;
  const int32_t* row_off;
  const int32_t* vlen;
  const int32_t* tokens;    // verify mode: drafted tokens [B, L]
  float* xg;                // verify mode: out, logit at the drafted token of each window row
  int64_t stride;
  int64_t rows;
  int B, L, K;
  int verify;
  int bonus;                // verify mode: 1 to include each request's bonus row (top-p filtering)
};

// Everything the accept/sample kernel reads and writes.
struct VerifyArgs {
  const void* target;
  const int32_t* row_off;
  const void* draft;
  const float* mix_w;       // nullable: w = 1 (K == 1)
  const int32_t* tokens;
  const int32_t* vlen;      // nullable
  const float* u;
  const float* g;
  int B, L, K;
  int64_t V;
  float T;
  int32_t* accept_len;
  int32_t* out_tokens;
  int* status;
  int* tickets;             // [B] blocks of each request finished, reset by the request's last block
  unsigned long long* keys; // [2B] best residual / bonus key per request, cleared by its last block
  const float* xg;          // [rows] logit at the drafted token (from the statistics kernel)
  const float2* rpart;      // row-statistics partials
  int G;                    // row-statistics grid size
  int64_t Vu;               // row-statistics units per row
  int P;                    // sampling blocks per request
  int topp;                 // rows filtered to their top-p nuclei: the fields below replace xg's partials
  const float* nuc_m;       // [walk rows] row maxima (walk with bonus rows)
  const double* nuc_lf;     // [walk rows] log nucleus masses
  const uint32_t* nuc_key;  // [walk rows] cut keys
  const int32_t* nuc_v;     // [walk rows] cut tokens
};

// The top-p nucleus kernel's inputs and outputs (one entry per walk row).
struct NucleusArgs {
  RowSpace rs;              // the verify walk, bonus rows included; xg receives the drafted-token logits
  int64_t V;
  float k;                  // log2(e) / T
  double top_p;
  float* row_m;             // out: row maximum (raw logit), NaN for a non-finite row
  double* row_lf;           // out: log of the nucleus mass sum_{v kept} 2^((x_v - m) k)
  uint32_t* cut_key;        // out: order key of the cut value
  int32_t* cut_v;           // out: cut token (tokens at the cut value with index <= cut_v are kept)
  int* flags;               // fast path, out: 1 for a row it hands to the exact kernel, else 0
  const int* only;          // exact kernel (nullable): process only the rows whose entry is non-zero
};

// Units of work per row: 16-byte vectors on the vector path, else elements.
inline int64_t units_per_row(int64_t V, int dtype, bool vec) {
  return vec ? V * (dtype == 0 ? 4 : 2) / 16 : V;
}

// Grid size of the row-statistics kernel for up to max_units units (Vu per row).
int stats_grid(int dtype, bool vec, int64_t max_units, int64_t Vu);

cudaError_t launch_row_stats(const RowSpace& rs, int dtype, bool vec, int64_t V, float T, int G,
                             float2* part, cudaStream_t st);

cudaError_t launch_softmax_finalize(const void* logits, int dtype, bool vec, int64_t rows, int64_t V,
                                    int64_t stride, float T, int G, const float2* part, float* row_max,
                                    float* row_lse, float* probs, cudaStream_t st);

cudaError_t launch_nucleus(const NucleusArgs& a, int dtype, bool vec, cudaStream_t st);
cudaError_t launch_nucleus_fast(const NucleusArgs& a, cudaStream_t st);  // bf16 rows of 16-byte vectors
constexpr int64_t kNucFastMinV = 4096;  // smaller rows take the exact kernel alone

cudaError_t launch_accept_sample(const VerifyArgs& a, int dtype, bool vec, cudaStream_t st);
int accept_blocks_per_sm(int dtype, bool vec, int K, bool topp);

cudaError_t launch_dvl(const float* scores, int B, int L, int budget, int32_t* verify_len,
                       int32_t* offsets, int32_t* slot_map, int* status, cudaStream_t st);

cudaError_t launch_pack(const void* dense, void* packed, int dtype, int B, int L, int64_t V,
                        int budget, const int32_t* offsets, cudaStream_t st);

// Launch helper: programmatic stream serialization lets the grid start while
// its predecessor drains; each kernel calls griddepcontrol.wait first.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

}  // namespace specv
