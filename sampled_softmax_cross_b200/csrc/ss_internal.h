// ss_internal.h -- declarations shared by the host API and the kernel files.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "ce_gemm.h"
#include "sampled_ce.h"

namespace ssb {

// Launches `kernel` on `s` with programmatic stream serialization: the grid may
// begin while the previous kernel on the stream is finishing. Every kernel of
// the library waits (griddepcontrol.wait) before its first global-memory
// access, so results are those of plain stream order.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t s, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// Small kernels (ce_kernels.cu). Each returns the launch error.
cudaError_t launch_build_mark(const int32_t* targets, int64_t T, int32_t V, int32_t P,
                              int64_t offset, int32_t stride, uint32_t* bitmap, int32_t* prefix,
                              int32_t* dev_status, cudaStream_t s);
cudaError_t launch_build_emit(const int32_t* targets, int64_t T, int32_t V, int32_t P,
                              const uint32_t* bitmap, const int32_t* prefix,
                              int32_t* dev_status, int32_t* candidates,
                              int32_t* target_pos, int32_t* vocab_pos, cudaStream_t s);
cudaError_t launch_gather(const uint16_t* lm_head, const int32_t* cand, int32_t P, int32_t d,
                          int32_t V, uint16_t* w_c, int32_t* status, int32_t* zero_words,
                          int32_t n_zero_words, cudaStream_t s);
// ref[i] = x_i . W_C[target_pos_i] (W_C[0] on ignored rows), fp32.
cudaError_t launch_ref_logits(const uint16_t* x, const uint16_t* w_c, const int32_t* tpos,
                              int64_t T, int32_t d, int32_t P, float* ref, cudaStream_t s);
// Row pass after the forward GEMM (see ce_kernels.cu).
struct RowArgs {
  const float* rowsum;  // [nsums][T] partial row sums of exp(z - ref)
  const float* ref;     // [T]
  const int32_t* tpos;  // [T]
  const uint16_t* x;    // [T][d]
  int64_t T;
  int32_t d, P, nsums;
  int64_t ldz;
  const uint16_t* w_c;  // [P][d] (fix-up)
  uint16_t* u;          // [T][ldz] E, patched at the target column
  float* lse;           // [T]
  float* rscale;        // [T]
  uint16_t* xs;         // [T][d] x' = rscale * x
  float* loss_rows;     // [T]
  int32_t* fix_list;    // [T] rows whose E overflowed
  int32_t* fix_count;   // [1]
  double2* partials;    // [kRowPartials] per-block (loss sum, valid count) of the row pass
  // e4m3 forward (nullptr otherwise): the fix-up recomputes logits from these
  const uint8_t* x8;    // [T][d] e4m3 codes of x
  const uint8_t* w8;    // [P][d] e4m3 codes of W_C
  const float* qscale;  // [3]: scale of x, of W_C, their product
  float* loss;          // [1] mean loss over valid rows
  int32_t* n_valid;     // [1]
  int32_t* status;      // dev_status + 8 (kernel error, detail)
};
// Most blocks the row pass launches (the size of RowArgs::partials).
constexpr int kRowPartials = 4096;
// Words of the workspace's counter block: the row pass's overflow count, the
// e4m3 amax pair, and the tile counters of the three GEMMs. The forward's
// gather zeroes all of them; dX zeroes dW's counter and dW zeroes dX's, so
// that a backward repeated after one forward starts from zero as well.
constexpr int kWordFixCount = 0, kWordAmax = 1, kWordFwdTiles = 4, kWordDxTiles = 5,
              kWordDwTiles = 6, kCounterWords = 8;
cudaError_t launch_rows(const RowArgs& a, cudaStream_t s);
// Exact recomputation of overflowed rows, then the loss mean (one CTA).
cudaError_t launch_finalize(const RowArgs& a, cudaStream_t s);
// prefix_pos[i] = position in C of prefix_table[targets[i]], -1 if none.
cudaError_t launch_prefix_pos(const int32_t* prefix_table, const int32_t* targets,
                              const int32_t* vocab_pos, int64_t T, int32_t V, int32_t* prefix_pos,
                              int32_t* status, cudaStream_t s);
// e4m3 quantization of one or two bf16 tensors (n, m multiples of 8 elements):
// amax[0..1] must be 0 before k_amax runs; qscale[0..2] = 2^ka, 2^kb, 2^(ka+kb).
cudaError_t launch_amax_bf16(const uint16_t* a, int64_t n, const uint16_t* b, int64_t m,
                             uint32_t* amax, cudaStream_t s);
cudaError_t launch_quant_e4m3(const uint16_t* a, int64_t n, uint8_t* a8, const uint16_t* b,
                              int64_t m, uint8_t* b8, const uint32_t* amax, float* qscale,
                              cudaStream_t s);
// ref[i] = qscale[2] * (x8_i . w8[target_pos_i]) in fp32 (w8[0] on ignored rows).
cudaError_t launch_ref_logits_e4m3(const uint8_t* x8, const uint8_t* w8, const int32_t* tpos,
                                   int64_t T, int32_t d, int32_t P, const float* qscale,
                                   float* ref, cudaStream_t s);
cudaError_t launch_zero_rows(uint16_t* dW, int32_t V, int32_t d, const int32_t* vocab_pos,
                             int all_rows, cudaStream_t s);

// Host side (ss_api.cu): the candidate build's two launches on caller-given
// scratch, and the error record behind ss_last_cuda_error.
ss_status enqueue_build(const int32_t* targets, int64_t T, int32_t V, int32_t P, int64_t offset,
                        int32_t stride, int32_t* candidates, int32_t* target_pos,
                        int32_t* vocab_pos, int32_t* dev_status, uint32_t* bitmap,
                        int32_t* prefix, cudaStream_t s);
ss_status record_cuda_error(cudaError_t e, const char* where);

}  // namespace ssb
