// ss_noalloc.cu -- ss_build_candidates_noalloc: the candidate build with its
// scratch memory in a fixed array inside the library, for callers that cannot
// hand the library a workspace.
//
// Who needs it: a caller whose device memory is owned by someone else and is
// fixed once set-up ends -- for example an inference or training server whose
// caching allocator has already reserved the device memory it is allowed to
// use, or a host-side hook that runs where allocating (cudaMalloc, or a
// framework allocator) is not permitted. Such a caller can still pass the
// input and output arrays it already owns, but cannot obtain the extra
// bitmap and prefix buffers the build needs. Here those live in a file-scope
// __device__ array: the CUDA runtime places it in device memory when the
// library is loaded, on every GPU that loads it, and it stays there until
// the process exits.
//
// The scratch is sized for the largest vocabulary the builder accepts
// (SS_MAX_VOCAB = 2^19 classes): a 2^19-bit class bitmap plus one int32 prefix
// per 32-bit bitmap word, 2 x 64 KB = 128 KB per device.
#include <mutex>

#include "ss_internal.h"

namespace {

constexpr int kWords = SS_MAX_VOCAB / 32;  // bitmap words for the largest V

// [0, kWords): class bitmap; [kWords, 2 * kWords): per-word prefix counts.
// Every call rewrites words [0, ceil(V/32)) of both halves before reading
// them, so nothing has to be cleared between calls.
static __device__ __align__(256) uint32_t g_build_scratch[2 * kWords];

std::mutex g_mu;
bool g_ready[128] = {};
uint32_t* g_scratch_ptr[128] = {};

// Device address of g_build_scratch on the current device. In host code the
// symbol names a host-side stand-in, not device memory, so the address must
// come from cudaGetSymbolAddress, once per device, with that device current.
// The address is kept for the life of the process: a process that destroys
// the device's primary context (cudaDeviceReset) must not call this entry
// point on that device again, since the array may then live elsewhere.
ss_status scratch_for_current_device(uint32_t** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return ssb::record_cuda_error(e, "cudaGetDevice");
  if (dev < 0 || dev >= 128) return SS_ERR_UNSUPPORTED_DEVICE;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_ready[dev]) {
    int major = 0;
    e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    if (e != cudaSuccess) return ssb::record_cuda_error(e, "cudaDeviceGetAttribute");
    if (major != 10) return SS_ERR_UNSUPPORTED_DEVICE;
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_build_scratch);
    if (e != cudaSuccess) return ssb::record_cuda_error(e, "cudaGetSymbolAddress");
    if (p == nullptr) return ssb::record_cuda_error(cudaErrorInvalidSymbol, "cudaGetSymbolAddress");
    g_scratch_ptr[dev] = static_cast<uint32_t*>(p);
    g_ready[dev] = true;
  }
  *out = g_scratch_ptr[dev];
  return SS_OK;
}

int gcd64(int64_t a, int64_t b) {
  while (b) {
    const int64_t t = a % b;
    a = b;
    b = t;
  }
  return (int)a;
}

}  // namespace

extern "C" SS_API ss_status ss_build_candidates_noalloc(
    const int32_t* targets, int64_t T, int32_t V, int32_t P, int64_t offset, int32_t stride,
    int32_t* candidates, int32_t* target_pos, int32_t* vocab_pos, int32_t* dev_status,
    void* stream) {
  // V above the size of the built-in scratch (SS_MAX_VOCAB) is rejected here.
  if (T < 0 || T > INT32_MAX || V < 1 || V > SS_MAX_VOCAB || P < 1 || P > V || offset < 0 ||
      stride < 1)
    return SS_ERR_INVALID_ARG;
  if (gcd64(stride, V) != 1) return SS_ERR_STRIDE_NOT_COPRIME;
  if ((T > 0 && (targets == nullptr || target_pos == nullptr)) || candidates == nullptr ||
      vocab_pos == nullptr || dev_status == nullptr)
    return SS_ERR_INVALID_ARG;
  if (T > 0 && (reinterpret_cast<uintptr_t>(targets) & 15u) != 0) return SS_ERR_MISALIGNED;
  uint32_t* scratch = nullptr;
  ss_status st = scratch_for_current_device(&scratch);
  if (st != SS_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint32_t* bitmap = scratch;
  int32_t* prefix = reinterpret_cast<int32_t*>(scratch + kWords);
  return ssb::enqueue_build(targets, T, V, P, offset, stride, candidates, target_pos, vocab_pos,
                            dev_status, bitmap, prefix, s);
}
