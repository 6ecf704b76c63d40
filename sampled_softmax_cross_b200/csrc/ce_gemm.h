// ce_gemm.h -- the interface of the tcgen05 GEMM kernels (ce_gemm.cu): their
// arguments, kinds and launch helpers.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ssb {

// Partial row sums the forward epilogue writes per 256-column tile: one per
// epilogue warp sharing a TMEM lane quarter (two, each over half of the
// tile's columns).
constexpr int kFwdSumsPerTileBf16 = 2, kFwdSumsPerTileE4m3 = 2;

// Arguments of the three tcgen05 GEMMs (forward logits, dX, dW_C).
struct GemmArgs {
  int32_t M, N, K;           // output rows, output cols, contraction length
  int32_t tiles_m, tiles_n;  // ceil(M / gemm_tile_rows(kind)), ceil(N / 256)
  int32_t num_kb;            // K blocks: ceil(K / 64), ceil(K / 128) for e4m3
  // forward epilogue: E = exp(z - ref) and its per-tile row sums
  const int32_t* tpos;  // [M] target position of each row, -1 = ignored
  const float* ref;     // [M] reference logit of each row
  const float* qscale;  // e4m3 forward: [2] = product of the two operand scales
  float* rowsum;        // [tiles_n * sums per tile][M] sums of exp(z - ref) over each
                        // tile, or over each half (128 columns) of it
  // dX / dW epilogue scale g / n (dX also times rscale[row])
  const float* grad_loss;
  const int32_t* n_valid;
  const float* rscale;  // [M] (dX) 1 / S_i, 0 on ignored rows
  // epilogues that store from registers (dX): output rows
  uint16_t* out;        // [M][ld_out] bf16 (dx; the forward's E when stored so)
  int64_t ld_out;
  // dW epilogue
  const int32_t* cand;       // [M] class id of each output row
  uint16_t* dW;              // [V][N] bf16
  int32_t V;
  const int32_t* vocab_pos;  // [V] (dW) rows with -1 are set to +0.0 by the epilogue warps
  int32_t* status;  // dev_status + 8 (error word, detail word)
  // dynamic tile schedule: this launch's tile counter (zero when it starts),
  // and a counter it sets to zero for the GEMM that follows it (or null)
  int32_t* tile_ctr;
  int32_t* next_ctr;
};

// KIND_FWD8: the forward on e4m3 operands (x and W_C quantized per tensor).
// KIND_DX, KIND_DW: 512-row tiles; KIND_DX1, KIND_DW1: the same GEMMs on
// 256-row tiles, for shapes where 512-row tiles would leave a poor last wave.
enum GemmKind { KIND_FWD = 0, KIND_DX = 1, KIND_DW = 2, KIND_FWD8 = 3, KIND_DX1 = 4, KIND_DW1 = 5 };
constexpr int kNumGemmKinds = 6;

// Launches `pairs` CTA pairs (clusters of 2) of the persistent GEMM kernel.
cudaError_t launch_gemm(int kind, const CUtensorMap& a, const CUtensorMap& b,
                        const CUtensorMap& c, const GemmArgs& args, int pairs, cudaStream_t s);
int gemm_smem_bytes(int kind);
// Output rows of one CTA pair's tile (256, or 512 where a tile takes two
// 128-row A blocks per CTA); GemmArgs::tiles_m counts tiles of this height.
int gemm_tile_rows(int kind);
const void* gemm_kernel_ptr(int kind);
int gemm_max_pairs(int kind, int sms);
// One CTA that runs the pipelines' bounded wait out on purpose (ce_gemm.cu).
cudaError_t launch_wait_selftest(int32_t* status, cudaStream_t s);

}  // namespace ssb
