// ss_internal.h -- declarations shared by the host API and the kernel files.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "sampled_ce.h"

namespace ssb {

// Arguments of the three tcgen05 GEMMs (forward logits, dX, dW_C).
struct GemmArgs {
  int32_t M, N, K;           // output rows, output cols, contraction length
  int32_t tiles_m, tiles_n;  // ceil(M / 256) (CTA-pair rows), ceil(N / 256)
  int32_t num_kb;            // ceil(K / 64)
  // forward epilogue
  const int32_t* tpos;  // [M] target position of each row, -1 = ignored
  float2* stats;        // [tiles_n][M] per-tile (row max, sum of exp(z - max))
  float* zt;            // [M] fp32 logit of the target column
  // forward converter warps: logits -> softmax - onehot, in place
  uint16_t* u;          // [M][ldz] bf16 logits, rewritten as softmax - onehot
  int64_t ldz;
  int32_t* done;        // [ceil(M / 128)] finished tiles per 128-row half-stripe
  int32_t* ticket;      // converter work-item counter
  float* lse;           // [M]
  double* partials;     // [2 * num_items] per work item: (sum of row losses, valid rows)
  int32_t num_items;    // ceil(M / kRowsPerItem)
  // dX / dW epilogue scale g / n
  const float* grad_loss;
  const int32_t* n_valid;
  // dW epilogue
  const int32_t* cand;  // [M] class id of each output row
  uint16_t* dW;         // [V][N] bf16
  int32_t V;
  int32_t* status;  // dev_status + 8 (error word, detail word)
};

constexpr int kRowsPerItem = 4;  // rows one converter warp takes at a time

enum GemmKind { KIND_FWD = 0, KIND_DX = 1, KIND_DW = 2 };

// Launches `pairs` CTA pairs (clusters of 2) of the persistent GEMM kernel.
cudaError_t launch_gemm(int kind, const CUtensorMap& a, const CUtensorMap& b,
                        const CUtensorMap& c, const GemmArgs& args, int pairs, cudaStream_t s);
int gemm_smem_bytes();
int gemm_rows_per_tile();
const void* gemm_kernel_ptr(int kind);
int gemm_max_pairs(int kind, int sms);

// Small kernels (ce_kernels.cu). Each returns the launch error.
cudaError_t launch_build_mark(const int32_t* targets, int64_t T, int32_t V, int32_t P,
                              int64_t offset, int32_t stride, uint32_t* bitmap, int32_t* prefix,
                              int32_t* dev_status, cudaStream_t s);
cudaError_t launch_build_emit(const int32_t* targets, int64_t T, int32_t V, int32_t P,
                              const uint32_t* bitmap, const int32_t* prefix,
                              const int32_t* dev_status, int32_t* candidates,
                              int32_t* target_pos, int32_t* vocab_pos, cudaStream_t s);
cudaError_t launch_gather(const uint16_t* lm_head, const int32_t* cand, int32_t P, int32_t d,
                          int32_t V, uint16_t* w_c, int32_t* status, int32_t* zero_words,
                          int32_t n_zero_words, cudaStream_t s);
cudaError_t launch_finalize(const double* partials, int32_t nitems, float* loss,
                            int32_t* n_valid, cudaStream_t s);
cudaError_t launch_zero_rows(uint16_t* dW, int32_t V, int32_t d, const int32_t* vocab_pos,
                             int all_rows, cudaStream_t s);

inline int converter_items(int64_t T) { return (int)((T + kRowsPerItem - 1) / kRowsPerItem); }

}  // namespace ssb
