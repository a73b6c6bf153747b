// Kernel argument blocks shared by the host code (zha_api.cu) and the
// decode / dense kernels.
#pragma once

#include "zha_common.cuh"

namespace zha {

struct DecodeArgs {
  TreeDev t;
  const void* Q;                // [nheads][d]: sequence-major, then query head
  float* O;                     // [nheads][d]
  int64_t n_tokens;
  int64_t nl[kMaxLevels + 1];   // complete nodes per level (nl[0] = tokens)
  int n_roots, n_steps;
  int nheads;                   // sequences x query heads of this call
  int max_heads;                // max_batch x query heads: the layout of the per-head scratch regions
  char* ws;                     // per-head workspaces, ws_per_bh bytes each
  uint64_t ws_per_bh;
  int64_t cap_sel;              // entries per step buffer (and kept parents)
  int64_t cap_list;             // kept leaves per head
  unsigned char* flow;          // per-head routing states, then leaf bitmaps (zero between launches)
  float* attn_part;             // attend partials, (2 + d) floats each
  long long spin_limit;         // bound of the waits on record copies
  int32_t* kept;
  int32_t* kept_cnt;
  int64_t* stats;
  int32_t* scored;
  int64_t scored_cap;
  int64_t kept_stride;
  // top-p threshold of routing step s (s = 0: the roots): p = p_mant[s] * 2^-p_shift[s] (p < 1);
  // p_all[s]: p >= 1, keep every candidate of the step
  uint32_t p_mant[kMaxLevels];
  int p_shift[kMaxLevels];
  int p_all[kMaxLevels];
  int root_gemm;                // the first routing step (the roots, shared by every query) as one contraction
};

struct DenseArgs {
  const void* K;
  const void* V;
  const void* Q;
  float* O;
  float* part;       // [B][Hq][splits][D + 2]
  int64_t ld;        // row stride of K / V in tokens
  int64_t n;
  int64_t per;       // keys per split (multiple of 64)
  int splits, hq, hkv, group;
  float inv_sqrt_d;
};

// kernels launched by this library (incremented by every launcher)
void count_launches(int n);

cudaError_t launch_decode(const DecodeArgs& a, int dtype, cudaStream_t st);
cudaError_t launch_dense(const DenseArgs& a, int dtype, int d, int B, cudaStream_t st);

}  // namespace zha
