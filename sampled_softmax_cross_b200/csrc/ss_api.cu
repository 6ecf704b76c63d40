// ss_api.cu -- the C ABI declared in include/sampled_ce.h: argument checks,
// workspace layout, TMA descriptors and the launch sequence of each call.
#include <cudaTypedefs.h>
#include <stdio.h>
#include <string.h>

#include <mutex>
#include <string>
#include <vector>

#include "ss_internal.h"

using namespace ssb;

namespace {

thread_local char g_last_error[512] = "";

ss_status cuda_fail(cudaError_t e, const char* where) {
  snprintf(g_last_error, sizeof(g_last_error), "%s: %s", where, cudaGetErrorString(e));
  return SS_ERR_CUDA;
}

#define SS_CUDA(call, where)                        \
  do {                                              \
    cudaError_t _e = (call);                        \
    if (_e != cudaSuccess) return cuda_fail(_e, where); \
  } while (0)

// ------------------------------------------------------------- device info --
struct DeviceState {
  bool ready = false;
  int sms = 0;
  int max_pairs[kNumGemmKinds] = {};  // resident CTA pairs of each GEMM kernel
  ss_status status = SS_OK;
};
std::mutex g_dev_mu;
DeviceState g_dev[128];

ss_status ensure_device(int* sms, int* max_pairs = nullptr) {
  int dev = 0;
  SS_CUDA(cudaGetDevice(&dev), "cudaGetDevice");
  if (dev < 0 || dev >= 128) return SS_ERR_UNSUPPORTED_DEVICE;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DeviceState& d = g_dev[dev];
  if (!d.ready) {
    int major = 0;
    SS_CUDA(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev),
            "cudaDeviceGetAttribute");
    SS_CUDA(cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev),
            "cudaDeviceGetAttribute");
    if (major != 10) {
      d.status = SS_ERR_UNSUPPORTED_DEVICE;
    } else {
      for (int k = 0; k < kNumGemmKinds; ++k) {
        SS_CUDA(cudaFuncSetAttribute(gemm_kernel_ptr(k),
                                     cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     gemm_smem_bytes(k)),
                "cudaFuncSetAttribute");
        d.max_pairs[k] = gemm_max_pairs(k, d.sms);
      }
    }
    d.ready = true;
  }
  *sms = d.sms;
  if (max_pairs != nullptr)
    for (int k = 0; k < kNumGemmKinds; ++k) max_pairs[k] = d.max_pairs[k];
  return d.status;
}

// --------------------------------------------------------------- TMA maps --
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D tensor [outer][inner] of bf16 (or, with elem_bytes 1, e4m3 codes) with
// row pitch `row_elems`, 128-byte swizzle.
ss_status make_map(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t outer,
                   uint64_t row_elems, uint32_t box_inner, uint32_t box_outer,
                   int elem_bytes = 2) {
  auto fn = encode_fn();
  if (fn == nullptr) {
    snprintf(g_last_error, sizeof(g_last_error), "cuTensorMapEncodeTiled unavailable");
    return SS_ERR_CUDA;
  }
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_elems * (uint64_t)elem_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, elem_bytes == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                  2, const_cast<void*>(ptr), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    snprintf(g_last_error, sizeof(g_last_error), "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return SS_ERR_CUDA;
  }
  return SS_OK;
}

// ----------------------------------------------------------------- timing --
struct TimingState {
  bool on = false;
  bool gemms_only = false;  // enable == 2: time only the tensor-core GEMM launches
  std::vector<cudaEvent_t> ev;        // pairs
  std::vector<int> rec_name;          // name index per used pair
  std::vector<std::string> names;
  size_t used = 0;
};
TimingState g_tm;
constexpr size_t kTimingPairs = 8192;

// Events are created when timing is switched on (ss_timing_enable), never
// inside a launch: creating thousands of events takes the host milliseconds,
// which inside a timed region would leave the GPU idle.
cudaError_t timing_make_events() {
  if (!g_tm.ev.empty()) return cudaSuccess;
  std::vector<cudaEvent_t> ev(2 * kTimingPairs);
  for (auto& e : ev) {
    const cudaError_t r = cudaEventCreate(&e);
    if (r != cudaSuccess) return r;
  }
  g_tm.ev.swap(ev);
  return cudaSuccess;
}

// `gemm`: the launch is one of the three tensor-core GEMMs (timed also in
// the GEMMs-only mode).
int timing_begin(const char* name, bool gemm, cudaStream_t s) {
  if (!g_tm.on || g_tm.ev.empty() || g_tm.used >= kTimingPairs) return -1;
  if (g_tm.gemms_only && !gemm) return -1;
  int idx = -1;
  for (size_t i = 0; i < g_tm.names.size(); ++i)
    if (g_tm.names[i] == name) idx = (int)i;
  if (idx < 0) {
    g_tm.names.push_back(name);
    idx = (int)g_tm.names.size() - 1;
  }
  const size_t slot = g_tm.used++;
  g_tm.rec_name.push_back(idx);
  cudaEventRecord(g_tm.ev[2 * slot], s);
  return (int)slot;
}

void timing_end(int slot, cudaStream_t s) {
  if (slot >= 0) cudaEventRecord(g_tm.ev[2 * slot + 1], s);
}

#define SS_LAUNCH_KIND(name, gemm, stream, call)              \
  do {                                                        \
    const int _slot = timing_begin(name, gemm, stream);       \
    cudaError_t _e = (call);                                  \
    timing_end(_slot, stream);                                \
    if (_e != cudaSuccess) return cuda_fail(_e, name);        \
  } while (0)
#define SS_LAUNCH(name, stream, call) SS_LAUNCH_KIND(name, false, stream, call)
#define SS_LAUNCH_GEMM(name, stream, call) SS_LAUNCH_KIND(name, true, stream, call)

// -------------------------------------------------------------- workspace --
constexpr int kBM = 128, kBN = 256;  // A rows per TMA box, output columns per tile

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

struct Layout {
  size_t bitmap, prefix, ref, rscale, loss_rows, fix_list, fix_count, partials, w_c, u, rowsum, xs,
      total;
  size_t x8, w8, qscale, total_e4m3;  // after `total`: the e4m3 forward's extra buffers
  int64_t ldz;
  int tiles_n;
};

bool sizes_ok(int64_t T, int32_t d, int32_t V, int32_t P) {
  return T >= 0 && T <= INT32_MAX && d >= 8 && d % 8 == 0 && d <= (1 << 16) && V >= 1 &&
         V <= SS_MAX_VOCAB && P >= 1 && P <= V;
}

Layout layout(int64_t T, int32_t d, int32_t V, int32_t P) {
  Layout L;
  const size_t nw = (size_t)(V + 31) / 32;
  L.ldz = (P + 7) / 8 * 8;
  L.tiles_n = (P + kBN - 1) / kBN;
  size_t off = 0;
  auto take = [&](size_t bytes, size_t align) {
    off = align_up(off, align);
    const size_t at = off;
    off += bytes;
    return at;
  };
  L.bitmap = take(nw * 4, 256);
  L.prefix = take(nw * 4, 256);
  L.ref = take((size_t)T * 4, 256);
  L.rscale = take((size_t)T * 4, 256);
  L.loss_rows = take((size_t)T * 4, 256);
  L.fix_list = take((size_t)T * 4, 256);
  L.fix_count = take(kCounterWords * 4, 256);
  L.partials = take((size_t)kRowPartials * sizeof(double2), 256);
  L.w_c = take((size_t)P * d * 2, 1024);
  L.u = take((size_t)T * L.ldz * 2, 1024);
  L.rowsum = take((size_t)L.tiles_n * kFwdSumsPerTileE4m3 * T * 4, 1024);  // the larger count
  L.xs = take((size_t)T * d * 2, 1024);
  L.total = align_up(off, 1024);
  off = L.total;
  L.x8 = take((size_t)T * d, 1024);
  L.w8 = take((size_t)P * d, 1024);
  L.qscale = take(16, 256);
  L.total_e4m3 = align_up(off, 1024);
  return L;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Tile height of a backward GEMM with M output rows and n_tiles 256-column
// tiles: 512-row tiles (`big`) load 25% fewer operand bytes per multiply-add
// and run about 5% faster per unit of work, 256-row tiles (`small`) come in
// twice the number and so fill the last wave of CTA pairs more evenly. The
// cost of each is its number of waves times the time of one of its tiles.
int backward_kind(int big, int small, int64_t M, int n_tiles, const int* pairs) {
  const int64_t t_big = (M + gemm_tile_rows(big) - 1) / gemm_tile_rows(big) * n_tiles;
  const int64_t t_small = (M + gemm_tile_rows(small) - 1) / gemm_tile_rows(small) * n_tiles;
  const int64_t w_big = (t_big + pairs[big] - 1) / pairs[big];
  const int64_t w_small = (t_small + pairs[small] - 1) / pairs[small];
  return 19 * w_big <= 10 * w_small ? big : small;  // a big tile ~ 1.9 small ones
}

int gcd_int(int64_t a, int64_t b) {
  while (b) {
    const int64_t t = a % b;
    a = b;
    b = t;
  }
  return (int)a;
}

}  // namespace

namespace ssb {

// The two builder launches, shared by ss_build_candidates and
// ss_build_candidates_noalloc (which differ only in where the bitmap and
// prefix scratch live). Launch errors go to ss_last_cuda_error and the
// launches are recorded by the kernel timer like every other launch.
ss_status enqueue_build(const int32_t* targets, int64_t T, int32_t V, int32_t P, int64_t offset,
                        int32_t stride, int32_t* candidates, int32_t* target_pos,
                        int32_t* vocab_pos, int32_t* dev_status, uint32_t* bitmap,
                        int32_t* prefix, cudaStream_t s) {
  SS_LAUNCH("build_mark", s,
            launch_build_mark(targets, T, V, P, offset % V, stride, bitmap, prefix, dev_status, s));
  SS_LAUNCH("build_emit", s,
            launch_build_emit(targets, T, V, P, bitmap, prefix, dev_status, candidates, target_pos,
                              vocab_pos, s));
  return SS_OK;
}

ss_status record_cuda_error(cudaError_t e, const char* where) { return cuda_fail(e, where); }

}  // namespace ssb

// ===================================================================== API ==
// The forward, with the logits GEMM on bf16 operands or (e4m3) on per-tensor
// e4m3 quantizations of x and W_C.
static ss_status forward_impl(const ss_bf16* x, const ss_bf16* lm_head,
                              const int32_t* candidates, const int32_t* target_pos, int64_t T,
                              int32_t d, int32_t V, int32_t P, float* loss, float* lse,
                              int32_t* n_valid, int32_t* dev_status, void* workspace,
                              size_t workspace_bytes, void* stream, bool e4m3) {
  if (!sizes_ok(T, d, V, P) || (e4m3 && d % 16 != 0)) return SS_ERR_INVALID_ARG;
  if (lm_head == nullptr || candidates == nullptr || loss == nullptr || n_valid == nullptr ||
      dev_status == nullptr || workspace == nullptr ||
      (T > 0 && (x == nullptr || target_pos == nullptr || lse == nullptr)))
    return SS_ERR_INVALID_ARG;
  if (!aligned16(lm_head) || !aligned16(workspace) || (T > 0 && !aligned16(x)))
    return SS_ERR_MISALIGNED;
  const Layout L = layout(T, d, V, P);
  if (workspace_bytes < (e4m3 ? L.total_e4m3 : L.total)) return SS_ERR_WORKSPACE_TOO_SMALL;
  int sms, pairs[kNumGemmKinds];
  ss_status ds = ensure_device(&sms, pairs);
  if (ds != SS_OK) return ds;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint16_t* w_c = reinterpret_cast<uint16_t*>(ws + L.w_c);
  uint16_t* u = reinterpret_cast<uint16_t*>(ws + L.u);
  float* ref = reinterpret_cast<float*>(ws + L.ref);
  float* rowsum = reinterpret_cast<float*>(ws + L.rowsum);
  float* loss_rows = reinterpret_cast<float*>(ws + L.loss_rows);
  int32_t* fix_count = reinterpret_cast<int32_t*>(ws + L.fix_count);
  int32_t* kstatus = dev_status + 8;

  RowArgs ra{};
  ra.rowsum = rowsum;
  ra.ref = ref;
  ra.tpos = target_pos;
  ra.x = x;
  ra.T = T;
  ra.d = d;
  ra.P = P;
  ra.nsums = L.tiles_n * (e4m3 ? kFwdSumsPerTileE4m3 : kFwdSumsPerTileBf16);
  ra.ldz = L.ldz;
  ra.w_c = w_c;
  ra.u = u;
  ra.lse = lse;
  ra.rscale = reinterpret_cast<float*>(ws + L.rscale);
  ra.xs = reinterpret_cast<uint16_t*>(ws + L.xs);
  ra.loss_rows = loss_rows;
  ra.fix_list = reinterpret_cast<int32_t*>(ws + L.fix_list);
  ra.fix_count = fix_count;
  ra.partials = reinterpret_cast<double2*>(ws + L.partials);
  ra.loss = loss;
  ra.n_valid = n_valid;
  ra.status = kstatus;
  uint8_t* x8 = ws + L.x8;
  uint8_t* w8 = ws + L.w8;
  float* qscale = reinterpret_cast<float*>(ws + L.qscale);
  uint32_t* amax = reinterpret_cast<uint32_t*>(fix_count + kWordAmax);  // zeroed with fix_count
  if (e4m3) {
    ra.x8 = x8;
    ra.w8 = w8;
    ra.qscale = qscale;
  }

  SS_LAUNCH("gather", s,
            launch_gather(lm_head, candidates, P, d, V, w_c, kstatus, fix_count, kCounterWords,
                          s));
  if (T > 0) {
    CUtensorMap ta, tb, tc;
    ss_status r;
    if (e4m3) {
      SS_LAUNCH("amax_e4m3", s, launch_amax_bf16(x, T * d, w_c, (int64_t)P * d, amax, s));
      SS_LAUNCH("quant_e4m3", s,
                launch_quant_e4m3(x, T * d, x8, w_c, (int64_t)P * d, w8, amax, qscale, s));
      SS_LAUNCH("ref_logits_e4m3", s,
                launch_ref_logits_e4m3(x8, w8, target_pos, T, d, P, qscale, ref, s));
      if ((r = make_map(&ta, x8, d, T, d, 128, kBM, 1)) != SS_OK) return r;
      if ((r = make_map(&tb, w8, d, P, d, 128, kBN / 2, 1)) != SS_OK) return r;
    } else {
      SS_LAUNCH("ref_logits", s, launch_ref_logits(x, w_c, target_pos, T, d, P, ref, s));
      if ((r = make_map(&ta, x, d, T, d, 64, kBM)) != SS_OK) return r;
      if ((r = make_map(&tb, w_c, d, P, d, 64, kBN / 2)) != SS_OK) return r;
    }
    if ((r = make_map(&tc, u, P, T, L.ldz, 64, 32)) != SS_OK) return r;
    GemmArgs a{};
    a.M = (int32_t)T;
    a.N = P;
    a.K = d;
    const int kind = e4m3 ? KIND_FWD8 : KIND_FWD;
    a.tiles_m = (int32_t)((T + gemm_tile_rows(kind) - 1) / gemm_tile_rows(kind));
    a.tiles_n = L.tiles_n;
    a.num_kb = e4m3 ? (d + 127) / 128 : (d + 63) / 64;
    a.tpos = target_pos;
    a.ref = ref;
    a.qscale = e4m3 ? qscale : nullptr;
    a.rowsum = rowsum;
    a.out = u;
    a.ld_out = L.ldz;
    a.status = kstatus;
    a.tile_ctr = fix_count + kWordFwdTiles;
    const int tiles = a.tiles_m * a.tiles_n;
    SS_LAUNCH_GEMM(e4m3 ? "fwd_gemm_ce_e4m3" : "fwd_gemm_ce", s,
              launch_gemm(kind, ta, tb, tc, a, tiles < pairs[kind] ? tiles : pairs[kind], s));
    SS_LAUNCH("row_pass", s, launch_rows(ra, s));
  }
  SS_LAUNCH("loss_finalize", s, launch_finalize(ra, s));
  return SS_OK;
}

extern "C" {

int32_t ss_version(void) { return 10000; }

const char* ss_last_cuda_error(void) { return g_last_error; }

const char* ss_status_string(int32_t s) {
  switch (s) {
    case SS_OK: return "ok";
    case SS_ERR_INVALID_ARG: return "invalid argument";
    case SS_ERR_BAD_TARGET: return "target outside [-1, V)";
    case SS_ERR_TOO_MANY_TARGETS: return "more distinct targets than candidates (D > P)";
    case SS_ERR_NO_FREE_CLASSES: return "not enough free classes for the negatives";
    case SS_ERR_STRIDE_NOT_COPRIME: return "stride not coprime with V";
    case SS_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case SS_ERR_MISALIGNED: return "pointer not 16-byte aligned";
    case SS_ERR_CUDA: return "CUDA runtime error";
    case SS_ERR_UNSUPPORTED_DEVICE: return "device is not sm_100 (B200)";
    case SS_ERR_KERNEL_TIMEOUT: return "kernel pipeline wait timed out";
    case SS_ERR_BAD_INDEX: return "candidate or position index out of range";
    default: return "unknown status";
  }
}

size_t ss_workspace_bytes(int64_t T, int32_t d, int32_t V, int32_t P) {
  if (!sizes_ok(T, d, V, P)) return 0;
  return layout(T, d, V, P).total;
}

size_t ss_workspace_wc_offset(int64_t T, int32_t d, int32_t V, int32_t P) {
  if (!sizes_ok(T, d, V, P)) return (size_t)-1;
  return layout(T, d, V, P).w_c;
}

size_t ss_build_workspace_bytes(int32_t V) {
  if (V < 1 || V > SS_MAX_VOCAB) return 0;
  return 2 * align_up((size_t)(V + 31) / 32 * 4, 256);
}

ss_status ss_build_candidates(const int32_t* targets, int64_t T, int32_t V, int32_t P,
                              int64_t offset, int32_t stride, int32_t* candidates,
                              int32_t* target_pos, int32_t* vocab_pos, int32_t* dev_status,
                              void* workspace, size_t workspace_bytes, void* stream) {
  if (T < 0 || T > INT32_MAX || V < 1 || V > SS_MAX_VOCAB || P < 1 || P > V || offset < 0 ||
      stride < 1)
    return SS_ERR_INVALID_ARG;
  if (gcd_int(stride, V) != 1) return SS_ERR_STRIDE_NOT_COPRIME;
  if ((T > 0 && targets == nullptr) || candidates == nullptr || vocab_pos == nullptr ||
      (T > 0 && target_pos == nullptr) || dev_status == nullptr || workspace == nullptr)
    return SS_ERR_INVALID_ARG;
  if ((T > 0 && !aligned16(targets)) || !aligned16(workspace)) return SS_ERR_MISALIGNED;
  const size_t nw = (size_t)(V + 31) / 32;
  if (workspace_bytes < ss_build_workspace_bytes(V)) return SS_ERR_WORKSPACE_TOO_SMALL;
  int sms;
  ss_status ds = ensure_device(&sms);
  if (ds != SS_OK) return ds;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint32_t* bitmap = reinterpret_cast<uint32_t*>(ws);
  int32_t* prefix = reinterpret_cast<int32_t*>(ws + align_up(nw * 4, 256));
  return enqueue_build(targets, T, V, P, offset, stride, candidates, target_pos, vocab_pos,
                       dev_status, bitmap, prefix, s);
}

ss_status ss_ce_forward(const ss_bf16* x, const ss_bf16* lm_head, const int32_t* candidates,
                        const int32_t* target_pos, int64_t T, int32_t d, int32_t V, int32_t P,
                        float* loss, float* lse, int32_t* n_valid, int32_t* dev_status,
                        void* workspace, size_t workspace_bytes, void* stream) {
  return forward_impl(x, lm_head, candidates, target_pos, T, d, V, P, loss, lse, n_valid,
                      dev_status, workspace, workspace_bytes, stream, false);
}

ss_status ss_ce_forward_e4m3(const ss_bf16* x, const ss_bf16* lm_head,
                             const int32_t* candidates, const int32_t* target_pos, int64_t T,
                             int32_t d, int32_t V, int32_t P, float* loss, float* lse,
                             int32_t* n_valid, int32_t* dev_status, void* workspace,
                             size_t workspace_bytes, void* stream) {
  return forward_impl(x, lm_head, candidates, target_pos, T, d, V, P, loss, lse, n_valid,
                      dev_status, workspace, workspace_bytes, stream, true);
}

size_t ss_workspace_bytes_e4m3(int64_t T, int32_t d, int32_t V, int32_t P) {
  if (!sizes_ok(T, d, V, P) || d % 16 != 0) return 0;
  return layout(T, d, V, P).total_e4m3;
}

ss_status ss_quantize_e4m3(const ss_bf16* src, int64_t n, uint8_t* dst, float* scale,
                           void* scratch, void* stream) {
  if (n < 0 || n % 8 != 0 || scale == nullptr || scratch == nullptr ||
      (n > 0 && (src == nullptr || dst == nullptr)))
    return SS_ERR_INVALID_ARG;
  if (!aligned16(src) || !aligned16(dst) || !aligned16(scratch)) return SS_ERR_MISALIGNED;
  int sms;
  ss_status ds = ensure_device(&sms);
  if (ds != SS_OK) return ds;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint32_t* amax = static_cast<uint32_t*>(scratch);      // words 0..1
  float* qs = static_cast<float*>(scratch) + 4;          // words 4..6
  SS_CUDA(cudaMemsetAsync(amax, 0, 2 * sizeof(uint32_t), s), "cudaMemsetAsync");
  SS_LAUNCH("amax_e4m3", s, launch_amax_bf16(src, n, nullptr, 0, amax, s));
  SS_LAUNCH("quant_e4m3", s, launch_quant_e4m3(src, n, dst, nullptr, 0, nullptr, amax, qs, s));
  SS_CUDA(cudaMemcpyAsync(scale, qs, sizeof(float), cudaMemcpyDeviceToDevice, s),
          "cudaMemcpyAsync");
  return SS_OK;
}

ss_status ss_ce_backward(const float* grad_loss, const int32_t* candidates,
                         const int32_t* vocab_pos, const int32_t* n_valid, int64_t T, int32_t d,
                         int32_t V, int32_t P, ss_bf16* dx, ss_bf16* dW, int32_t* dev_status,
                         void* workspace, size_t workspace_bytes, void* stream) {
  if (!sizes_ok(T, d, V, P)) return SS_ERR_INVALID_ARG;
  if (grad_loss == nullptr || candidates == nullptr || vocab_pos == nullptr ||
      n_valid == nullptr || dW == nullptr || dev_status == nullptr || workspace == nullptr ||
      (T > 0 && dx == nullptr))
    return SS_ERR_INVALID_ARG;
  if (!aligned16(dW) || !aligned16(workspace) || (T > 0 && !aligned16(dx)))
    return SS_ERR_MISALIGNED;
  const Layout L = layout(T, d, V, P);
  if (workspace_bytes < L.total) return SS_ERR_WORKSPACE_TOO_SMALL;
  int sms, pairs[kNumGemmKinds];
  ss_status ds = ensure_device(&sms, pairs);
  if (ds != SS_OK) return ds;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint16_t* w_c = reinterpret_cast<uint16_t*>(ws + L.w_c);
  uint16_t* u = reinterpret_cast<uint16_t*>(ws + L.u);
  uint16_t* xs = reinterpret_cast<uint16_t*>(ws + L.xs);
  int32_t* counters = reinterpret_cast<int32_t*>(ws + L.fix_count);
  int32_t* kstatus = dev_status + 8;

  if (T == 0) {
    SS_LAUNCH("zero_rows", s, launch_zero_rows(dW, V, d, vocab_pos, 1, s));
    return SS_OK;
  }

  CUtensorMap ua, wb, dxs, ua2, xb;
  ss_status r;
  if ((r = make_map(&ua, u, P, T, L.ldz, 64, kBM)) != SS_OK) return r;   // E', K-major
  if ((r = make_map(&wb, w_c, d, P, d, 64, 64)) != SS_OK) return r;      // W_C, MN-major
  if ((r = make_map(&dxs, dx, d, T, d, 64, 32)) != SS_OK) return r;      // dx store
  if ((r = make_map(&ua2, u, P, T, L.ldz, 64, 64)) != SS_OK) return r;   // E'^T, MN-major
  if ((r = make_map(&xb, xs, d, T, d, 64, 64)) != SS_OK) return r;       // x', MN-major

  const int n_tiles = (d + kBN - 1) / kBN;
  const int kdx = backward_kind(KIND_DX, KIND_DX1, T, n_tiles, pairs);
  const int kdw = backward_kind(KIND_DW, KIND_DW1, P, n_tiles, pairs);
  GemmArgs a{};
  a.M = (int32_t)T;
  a.N = d;
  a.K = P;
  a.tiles_m = (int32_t)((T + gemm_tile_rows(kdx) - 1) / gemm_tile_rows(kdx));
  a.tiles_n = n_tiles;
  a.num_kb = (P + 63) / 64;
  a.grad_loss = grad_loss;
  a.n_valid = n_valid;
  a.rscale = reinterpret_cast<const float*>(ws + L.rscale);
  a.out = dx;
  a.ld_out = d;
  a.status = kstatus;
  a.tile_ctr = counters + kWordDxTiles;
  a.next_ctr = counters + kWordDwTiles;
  const int tiles = a.tiles_m * a.tiles_n;
  SS_LAUNCH_GEMM("dx_gemm", s,
            launch_gemm(kdx, ua, wb, dxs, a, tiles < pairs[kdx] ? tiles : pairs[kdx], s));

  GemmArgs b{};
  b.M = P;
  b.N = d;
  b.K = (int32_t)T;
  b.tiles_m = (P + gemm_tile_rows(kdw) - 1) / gemm_tile_rows(kdw);
  b.tiles_n = n_tiles;
  b.num_kb = (int32_t)((T + 63) / 64);
  b.cand = candidates;
  b.dW = dW;
  b.V = V;
  b.vocab_pos = vocab_pos;  // the epilogue warps also zero the rows outside C
  b.grad_loss = grad_loss;
  b.n_valid = n_valid;
  b.status = kstatus;
  b.tile_ctr = counters + kWordDwTiles;
  b.next_ctr = counters + kWordDxTiles;
  // every resident pair, even without a tile, so that the zero rows are spread over all SMs
  SS_LAUNCH_GEMM("dw_gemm_scatter", s, launch_gemm(kdw, ua2, xb, ua2, b, pairs[kdw], s));
  return SS_OK;
}

ss_status ss_prefix_positions(const int32_t* prefix_table, const int32_t* targets,
                              const int32_t* vocab_pos, int64_t T, int32_t V, int32_t* prefix_pos,
                              int32_t* dev_status, void* stream) {
  if (T < 0 || T > INT32_MAX || V < 1 || V > SS_MAX_VOCAB) return SS_ERR_INVALID_ARG;
  if (prefix_table == nullptr || vocab_pos == nullptr || dev_status == nullptr ||
      (T > 0 && (targets == nullptr || prefix_pos == nullptr)))
    return SS_ERR_INVALID_ARG;
  int sms;
  ss_status ds = ensure_device(&sms);
  if (ds != SS_OK) return ds;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  SS_LAUNCH("prefix_pos", s,
            launch_prefix_pos(prefix_table, targets, vocab_pos, T, V, prefix_pos, dev_status + 8, s));
  return SS_OK;
}

ss_status ss_selftest_wait_limit(int32_t* dev_status, void* stream) {
  if (dev_status == nullptr) return SS_ERR_INVALID_ARG;
  int sms;
  ss_status ds = ensure_device(&sms);
  if (ds != SS_OK) return ds;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  SS_LAUNCH("wait_selftest", s, launch_wait_selftest(dev_status + 8, s));
  return SS_OK;
}

ss_status ss_timing_enable(int32_t enable) {
  if (enable != 0) SS_CUDA(timing_make_events(), "cudaEventCreate");
  g_tm.on = enable != 0;
  g_tm.gemms_only = enable == 2;
  return SS_OK;
}

ss_status ss_timing_reset(void) {
  g_tm.used = 0;
  g_tm.rec_name.clear();
  g_tm.names.clear();
  return SS_OK;
}

int32_t ss_timing_count(void) { return (int32_t)g_tm.names.size(); }

ss_status ss_timing_query(int32_t i, char* name, int32_t name_len, int32_t* launches,
                          double* total_ms) {
  if (i < 0 || i >= (int32_t)g_tm.names.size()) return SS_ERR_INVALID_ARG;
  if (name != nullptr && name_len > 0) {
    strncpy(name, g_tm.names[i].c_str(), (size_t)name_len - 1);
    name[name_len - 1] = '\0';
  }
  int n = 0;
  double tot = 0.0;
  for (size_t k = 0; k < g_tm.used; ++k) {
    if (g_tm.rec_name[k] != i) continue;
    SS_CUDA(cudaEventSynchronize(g_tm.ev[2 * k + 1]), "cudaEventSynchronize");
    float ms = 0.f;
    SS_CUDA(cudaEventElapsedTime(&ms, g_tm.ev[2 * k], g_tm.ev[2 * k + 1]), "cudaEventElapsedTime");
    tot += ms;
    ++n;
  }
  if (launches) *launches = n;
  if (total_ms) *total_ms = tot;
  return SS_OK;
}

}  // extern "C"
