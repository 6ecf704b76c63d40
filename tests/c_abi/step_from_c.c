/*
 * One build + forward + backward through the C ABI from a plain C99 program:
 * the boundary needs no Python and no C++. Device memory comes from the CUDA
 * runtime; the library allocates nothing.
 *
 * usage: step_from_c IN OUT T d V P offset
 *   IN : x [T*d] bf16 bits, lm_head [V*d] bf16 bits, targets [T] int32
 *   OUT: loss f32, n_valid i32, dev_status [16] i32, candidates [P] i32,
 *        target_pos [T] i32, dx [T*d] bf16 bits, dW [V*d] bf16 bits
 */
#include <stdio.h>
#include <stdlib.h>

#include <cuda_runtime_api.h>

#include "sampled_ce.h"

#define CK(call)                                                               \
  do {                                                                         \
    cudaError_t e_ = (call);                                                   \
    if (e_ != cudaSuccess) {                                                   \
      fprintf(stderr, "%s: %s\n", #call, cudaGetErrorString(e_));              \
      return 2;                                                                \
    }                                                                          \
  } while (0)

#define SS(call)                                                               \
  do {                                                                         \
    ss_status s_ = (call);                                                     \
    if (s_ != SS_OK) {                                                         \
      fprintf(stderr, "%s: %s\n", #call, ss_status_string(s_));               \
      return 3;                                                                \
    }                                                                          \
  } while (0)

static int read_all(FILE* f, void* p, size_t n) { return fread(p, 1, n, f) == n; }
static int write_all(FILE* f, const void* p, size_t n) { return fwrite(p, 1, n, f) == n; }

int main(int argc, char** argv) {
  if (argc != 8) {
    fprintf(stderr, "usage: %s IN OUT T d V P offset\n", argv[0]);
    return 1;
  }
  const long long T = atoll(argv[3]);
  const int d = atoi(argv[4]), V = atoi(argv[5]), P = atoi(argv[6]);
  const long long offset = atoll(argv[7]);
  const size_t nx = (size_t)T * d, nw = (size_t)V * d;

  uint16_t* hx = malloc(nx * 2);
  uint16_t* hlm = malloc(nw * 2);
  int32_t* ht = malloc((size_t)T * 4);
  FILE* fin = fopen(argv[1], "rb");
  if (!fin || !hx || !hlm || !ht || !read_all(fin, hx, nx * 2) || !read_all(fin, hlm, nw * 2) ||
      !read_all(fin, ht, (size_t)T * 4)) {
    fprintf(stderr, "cannot read %s\n", argv[1]);
    return 1;
  }
  fclose(fin);

  const size_t ws_bytes = ss_workspace_bytes(T, d, V, P);
  if (ws_bytes == 0) {
    fprintf(stderr, "invalid sizes\n");
    return 1;
  }
  void *x, *lm, *t, *cand, *tpos, *vpos, *st, *loss, *lse, *nv, *g, *dx, *dW, *ws;
  CK(cudaMalloc(&x, nx * 2));
  CK(cudaMalloc(&lm, nw * 2));
  CK(cudaMalloc(&t, (size_t)T * 4));
  CK(cudaMalloc(&cand, (size_t)P * 4));
  CK(cudaMalloc(&tpos, (size_t)T * 4));
  CK(cudaMalloc(&vpos, (size_t)V * 4));
  CK(cudaMalloc(&st, SS_DEV_STATUS_WORDS * 4));
  CK(cudaMalloc(&loss, 4));
  CK(cudaMalloc(&lse, (size_t)T * 4));
  CK(cudaMalloc(&nv, 4));
  CK(cudaMalloc(&g, 4));
  CK(cudaMalloc(&dx, nx * 2));
  CK(cudaMalloc(&dW, nw * 2));
  CK(cudaMalloc(&ws, ws_bytes));
  const float one = 1.0f;
  CK(cudaMemcpy(x, hx, nx * 2, cudaMemcpyHostToDevice));
  CK(cudaMemcpy(lm, hlm, nw * 2, cudaMemcpyHostToDevice));
  CK(cudaMemcpy(t, ht, (size_t)T * 4, cudaMemcpyHostToDevice));
  CK(cudaMemcpy(g, &one, 4, cudaMemcpyHostToDevice));
  CK(cudaMemset(st, 0, SS_DEV_STATUS_WORDS * 4));

  SS(ss_build_candidates(t, T, V, P, offset, SS_DEFAULT_STRIDE, cand, tpos, vpos, st, ws,
                         ws_bytes, NULL));
  SS(ss_ce_forward(x, lm, cand, tpos, T, d, V, P, loss, lse, nv, st, ws, ws_bytes, NULL));
  SS(ss_ce_backward(g, cand, vpos, nv, T, d, V, P, dx, dW, st, ws, ws_bytes, NULL));
  CK(cudaDeviceSynchronize());

  float hloss;
  int32_t hnv, hst[SS_DEV_STATUS_WORDS];
  int32_t* hcand = malloc((size_t)P * 4);
  int32_t* htpos = malloc((size_t)T * 4);
  uint16_t* hdx = malloc(nx * 2);
  uint16_t* hdW = malloc(nw * 2);
  if (!hcand || !htpos || !hdx || !hdW) return 1;
  CK(cudaMemcpy(&hloss, loss, 4, cudaMemcpyDeviceToHost));
  CK(cudaMemcpy(&hnv, nv, 4, cudaMemcpyDeviceToHost));
  CK(cudaMemcpy(hst, st, sizeof(hst), cudaMemcpyDeviceToHost));
  CK(cudaMemcpy(hcand, cand, (size_t)P * 4, cudaMemcpyDeviceToHost));
  CK(cudaMemcpy(htpos, tpos, (size_t)T * 4, cudaMemcpyDeviceToHost));
  CK(cudaMemcpy(hdx, dx, nx * 2, cudaMemcpyDeviceToHost));
  CK(cudaMemcpy(hdW, dW, nw * 2, cudaMemcpyDeviceToHost));

  FILE* fout = fopen(argv[2], "wb");
  if (!fout || !write_all(fout, &hloss, 4) || !write_all(fout, &hnv, 4) ||
      !write_all(fout, hst, sizeof(hst)) || !write_all(fout, hcand, (size_t)P * 4) ||
      !write_all(fout, htpos, (size_t)T * 4) || !write_all(fout, hdx, nx * 2) ||
      !write_all(fout, hdW, nw * 2)) {
    fprintf(stderr, "cannot write %s\n", argv[2]);
    return 1;
  }
  fclose(fout);
  printf("loss %.6f n_valid %d status %d\n", hloss, hnv, hst[0]);
  return 0;
}
