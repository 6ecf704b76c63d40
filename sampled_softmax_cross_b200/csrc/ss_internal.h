// ss_internal.h -- declarations shared by the host API and the kernel files.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/sampled_ce.h"

namespace ssb {

// Arguments of the three tcgen05 GEMMs (forward logits, dX, dW_C).
struct GemmArgs {
  int32_t M, N, K;           // output rows, output cols, contraction length
  int32_t tiles_m, tiles_n;  // ceil(M / 128), ceil(N / 256)
  int32_t num_kb;            // ceil(K / 64)
  // forward epilogue
  const int32_t* tpos;  // [M] target position of each row, -1 = ignored
  float2* stats;        // [tiles_n][M] per-tile (row max, sum of exp(z - max))
  float* zt;            // [M] fp32 logit of the target column
  // dW epilogue
  const int32_t* cand;  // [M] class id of each output row
  uint16_t* dW;         // [V][N] bf16
  int32_t V;
  int32_t* status;  // dev_status + 8 (error word, detail word)
};

enum GemmKind { KIND_FWD = 0, KIND_DX = 1, KIND_DW = 2 };

cudaError_t launch_gemm(int kind, const CUtensorMap& a, const CUtensorMap& b,
                        const CUtensorMap& c, const GemmArgs& args, int grid, cudaStream_t s);
int gemm_smem_bytes();
const void* gemm_kernel_ptr(int kind);

// Small kernels (ce_kernels.cu). Each returns the launch error.
cudaError_t launch_build_mark(const int32_t* targets, int64_t T, int32_t V, int32_t P,
                              int64_t offset, int32_t stride, uint32_t* bitmap, int32_t* prefix,
                              int32_t* dev_status, cudaStream_t s);
cudaError_t launch_build_emit(const int32_t* targets, int64_t T, int32_t V, int32_t P,
                              const uint32_t* bitmap, const int32_t* prefix,
                              const int32_t* dev_status, int32_t* candidates,
                              int32_t* target_pos, int32_t* vocab_pos, cudaStream_t s);
cudaError_t launch_gather(const uint16_t* lm_head, const int32_t* cand, int32_t P, int32_t d,
                          int32_t V, uint16_t* w_c, int32_t* status, cudaStream_t s);
cudaError_t launch_combine(const float2* stats, const float* zt, const int32_t* tpos, int64_t T,
                           int32_t P, int32_t tiles_n, float* lse, double* partials,
                           int32_t nblocks, cudaStream_t s);
cudaError_t launch_finalize(const double* partials, int32_t nblocks, float* loss,
                            int32_t* n_valid, cudaStream_t s);
cudaError_t launch_dlogits(uint16_t* z, int64_t T, int32_t P, int64_t ldz, const float* lse,
                           const int32_t* tpos, const float* grad_loss, const int32_t* n_valid,
                           cudaStream_t s);
cudaError_t launch_zero_rows(uint16_t* dW, int32_t V, int32_t d, const int32_t* vocab_pos,
                             int all_rows, cudaStream_t s);

constexpr int kCombineThreads = 256;
inline int combine_blocks(int64_t T) {
  return (int)((T + kCombineThreads - 1) / kCombineThreads);
}

}  // namespace ssb
