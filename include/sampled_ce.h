/*
 * sampled_ce.h -- C ABI of the B200 (sm_100a) shared-negatives sampled-softmax
 * cross-entropy LM head: candidate build, forward and backward.
 *
 * The method is the one of "sampled_softmax.py" (modded-nanogpt,
 * track_1_short): all tokens of a microbatch use one candidate set C of P
 * classes -- the classes that occur as targets in the microbatch, topped up
 * with negatives read from the stride permutation k * stride mod V, a window
 * that moves on every build -- and the cross-entropy normalises over C rather than the
 * whole vocabulary (module docstring, "What"). The lm_head gradient covers
 * all V rows, with exact zeros in the rows of classes not in C.
 *
 * Conventions for every entry point
 *   - All array arguments are DEVICE pointers on the current CUDA device,
 *     row-major and contiguous, 16-byte aligned. bf16 values are passed as
 *     their raw 16-bit patterns (ss_bf16).
 *   - The caller owns every buffer, the workspace included. The library
 *     allocates no device memory and keeps no state between calls, apart
 *     from per-device launch attributes it sets once.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream). All work
 *     is enqueued on it; no call synchronises the device. Kernels are
 *     launched with programmatic stream serialization: each may begin while
 *     the previous kernel on the stream finishes, and waits for it to complete
 *     before touching global memory, so results are those of plain stream
 *     order (a caller's own kernels launched normally are unaffected).
 *   - Host-detectable errors (sizes, alignment, workspace too small, a
 *     stride not coprime with V, a device that is not sm_100) return a
 *     non-zero ss_status before anything is enqueued. Errors that only the
 *     device can see are written to `dev_status` (below); read it after the
 *     stream has reached the call.
 *   - Index types are int32 (V < 2^31). The ignore marker for a target is -1.
 *
 * dev_status: int32[SS_DEV_STATUS_WORDS], device memory. ss_build_candidates
 * rewrites all 16 words; ss_ce_forward and ss_ce_backward only ever set
 * words 8..9 (first error wins), so one buffer can serve a whole step.
 *   [0] builder status (ss_status)      [1] D: distinct valid targets
 *   [2] need = P - D                    [3] 1 if the fallback pick ran
 *   [4] draw: window positions consumed [5] next offset = (offset + draw) mod V
 *   [6] first token index with a bad target, else -1
 *   [7] number of classes marked (P when the build succeeded)
 *   [8] forward/backward kernel error (ss_status, 0 = none)
 *   [9] detail for [8] (kernel id)      [10..11] written by
 *   ss_selftest_wait_limit only          [12..15] reserved (0)
 */
#ifndef SAMPLED_CE_H
#define SAMPLED_CE_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SS_API __attribute__((visibility("default")))
#else
#define SS_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t ss_bf16; /* raw bfloat16 bits */

typedef enum ss_status {
  SS_OK = 0,
  SS_ERR_INVALID_ARG = 1,        /* a size or pointer argument is out of range */
  SS_ERR_BAD_TARGET = 2,         /* a target outside [-1, V) (device) */
  SS_ERR_TOO_MANY_TARGETS = 3,   /* D > P distinct targets (device) */
  SS_ERR_NO_FREE_CLASSES = 4,    /* fewer than P - D classes left (device) */
  SS_ERR_STRIDE_NOT_COPRIME = 5, /* gcd(stride, V) != 1 */
  SS_ERR_WORKSPACE_TOO_SMALL = 6,
  SS_ERR_MISALIGNED = 7,         /* a pointer is not 16-byte aligned */
  SS_ERR_CUDA = 8,               /* a CUDA runtime call failed; see ss_last_cuda_error */
  SS_ERR_UNSUPPORTED_DEVICE = 9, /* the current device is not compute capability 10.x */
  SS_ERR_KERNEL_TIMEOUT = 10,    /* a pipeline wait ran out of time (device) */
  SS_ERR_BAD_INDEX = 11          /* a candidate or position outside its range (device) */
} ss_status;

#define SS_DEV_STATUS_WORDS 16
#define SS_DEFAULT_STRIDE 20011 /* NEGATIVE_STRIDE of sampled_softmax.py */
#define SS_MAX_VOCAB (1 << 19)  /* largest V the candidate builder accepts */

/* Bytes of workspace the three calls need for these sizes (0 if the sizes
 * are invalid). One workspace serves ss_build_candidates, ss_ce_forward and
 * ss_ce_backward of the same microbatch; ss_ce_forward leaves the gathered
 * rows W_C and the gradient factors (below) in it for ss_ce_backward, so it must not be
 * reused between a forward and its backward (sampled_softmax.py,
 * SampledSoftmax.__init__, keeps the same rule: a single microbatch in flight
 * per step). */
SS_API size_t ss_workspace_bytes(int64_t T, int32_t d, int32_t V, int32_t P);

/* Byte offset, inside that workspace, of the gathered rows W_C = lm_head[C]
 * ([P, d] bf16, row-major, row pitch d) that ss_ce_forward and
 * ss_ce_forward_e4m3 leave there for the backward (sampled_softmax.py,
 * SampledSoftmax._gather_rows: a plain row copy, so W_C can be checked bit
 * for bit against lm_head[C]). Returns (size_t)-1 if the sizes are invalid.
 * Read-only diagnostics: the rows are valid once the stream has passed the
 * forward and until the workspace is next used. */
SS_API size_t ss_workspace_wc_offset(int64_t T, int32_t d, int32_t V, int32_t P);

/* Bytes of workspace ss_build_candidates alone needs for a vocabulary of V
 * classes (0 if V is out of range). ss_workspace_bytes covers it as well. */
SS_API size_t ss_build_workspace_bytes(int32_t V);

/* Candidate set C for one microbatch.
 * sampled_softmax.py, CandidateBuilder.build and CandidateBuilder._negatives:
 *   mark every valid target; D = number of marked classes (D > P is an error);
 *   if D < P take need = P - D negatives: the first `need` unmarked classes of
 *   the stride sweep c_k = (stride * k) mod V for k = offset, offset+1, ...,
 *   offset+draw-1 (k mod V), draw = min(V, floor(1.7 * need) + 256); if that
 *   window holds fewer than `need` unmarked classes, take instead every s-th
 *   ascending unmarked class from the first, s = max(1, #unmarked / need).
 *   C = marked classes in ascending order.
 * In:  targets [T] int32, each in [-1, V) (-1 = ignored token);
 *      offset >= 0 (reduced mod V); stride coprime with V (SS_DEFAULT_STRIDE).
 *      1 <= P <= V <= SS_MAX_VOCAB, T >= 0.
 * Out: candidates [P] int32 ascending class ids;
 *      target_pos [T] int32: position of targets[i] in C, -1 for ignored;
 *      vocab_pos  [V] int32: position of each class in C, -1 outside C;
 *      dev_status [16] (see above). On a device-detected error the three
 *      arrays are filled with -1. */
SS_API ss_status ss_build_candidates(const int32_t* targets, int64_t T, int32_t V, int32_t P,
                              int64_t offset, int32_t stride, int32_t* candidates,
                              int32_t* target_pos, int32_t* vocab_pos, int32_t* dev_status,
                              void* workspace, size_t workspace_bytes, void* stream);

/* Allocation-free variant of ss_build_candidates. The pages the method comes
 * from have no counterpart: it exists for callers that cannot give the
 * library a workspace -- callers whose device memory is fixed once their
 * set-up ends (a server or trainer whose caching allocator already holds all
 * the memory it may use, a hook that must not allocate). They own the input
 * and output arrays but cannot provide the extra scratch buffers.
 * Same arguments (minus the workspace), results and dev_status as
 * ss_build_candidates. The call allocates nothing: the bitmap and prefix
 * scratch lives in a fixed 128 KB array inside the library, sized for
 * V <= SS_MAX_VOCAB (a larger V returns SS_ERR_INVALID_ARG), present on every
 * GPU that loads the library until the process exits.
 * The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress) with that device current; make that first call
 * before any stream capture. The address is then kept for the life of the
 * process: after cudaDeviceReset on a device, do not call this entry point
 * on that device again in the same process. All calls on a device share the one array:
 * calls whose work overlaps on the GPU (two streams, or two host threads
 * without ordering) race and give wrong results, so order them on one
 * stream. Each call rewrites every part of the array it reads, so nothing
 * needs clearing between calls. */
SS_API ss_status ss_build_candidates_noalloc(const int32_t* targets, int64_t T, int32_t V,
                                             int32_t P, int64_t offset, int32_t stride,
                                             int32_t* candidates, int32_t* target_pos,
                                             int32_t* vocab_pos, int32_t* dev_status,
                                             void* stream);

/* Forward: W_C = lm_head[C] (sampled_softmax.py, SampledSoftmax._gather_rows),
 * logits z = x @ W_C^T with fp32 accumulation, and an online-softmax
 * cross-entropy over the P columns ("Learning Triton One Kernel at a Time:
 * Softmax", section "Online Softmax"):
 *   lse[i]  = log sum_j exp(z_ij), for every row (ignored rows included);
 *   loss    = sum over valid rows of (lse[i] - z[i, target_pos[i]]) / n_valid,
 *             0 when n_valid = 0 (token-weighted mean, as in Handout #16's
 *             lm_gradient);
 *   n_valid = number of rows with target_pos >= 0.
 * The forward also leaves in the workspace what the backward needs for the
 * loss gradient w.r.t. the logits (section "Gradient": softmax minus one-hot):
 * E'_ij = exp(z_ij - z_i,target) (bf16; 1 - S_i at the target column, S_i the
 * row sum), r_i = 1 / S_i and x'_i = r_i x_i, so that r_i E'_ij equals
 * softmax_ij - [j == target_pos_i]; ignored rows have r_i = 0 and x'_i = 0.
 * In:  x [T, d] bf16; lm_head [V, d] bf16; candidates [P], target_pos [T] as
 *      written by ss_build_candidates. d % 8 == 0.
 * Out: loss [1] float32, lse [T] float32, n_valid [1] int32.
 * Workspace: keeps W_C [P, d], E' [T, P] and x' [T, d] (bf16) for the backward. */
SS_API ss_status ss_ce_forward(const ss_bf16* x, const ss_bf16* lm_head, const int32_t* candidates,
                        const int32_t* target_pos, int64_t T, int32_t d, int32_t V, int32_t P,
                        float* loss, float* lse, int32_t* n_valid, int32_t* dev_status,
                        void* workspace, size_t workspace_bytes, void* stream);

/* The forward above with the logits GEMM on 8-bit floating-point operands,
 * as sampled_softmax.py keeps them (SampledLoss.rows: the candidate rows in
 * float8 e4m3, fed to torch._scaled_mm). Format: OCP 8-bit floating point
 * E4M3 (4 exponent bits, bias 7, 3 mantissa bits, largest finite 448).
 * The pages give no scales; here each of x and W_C gets one power-of-two
 * scale 2^k, the smallest with max|v| * 2^-k <= 448 (k in [-126, 127]), and
 * the codes are v * 2^-k rounded to nearest even, saturating at +-448. The
 * logits are z = 2^(kx + kw) (x_q . W_C,q) with fp32 accumulation on the
 * tcgen05 tensor cores (kind::f8f6f4); lse, the loss and the gradient
 * factors follow from that z exactly as in ss_ce_forward, so ss_ce_backward
 * (bf16 gradient GEMMs on x and W_C) runs unchanged after it.
 * Arguments as ss_ce_forward; additionally d % 16 == 0 and the workspace
 * holds ss_workspace_bytes_e4m3(T, d, V, P) bytes (the bf16 layout plus the
 * codes of x and W_C at its end). */
SS_API ss_status ss_ce_forward_e4m3(const ss_bf16* x, const ss_bf16* lm_head,
                                    const int32_t* candidates, const int32_t* target_pos,
                                    int64_t T, int32_t d, int32_t V, int32_t P, float* loss,
                                    float* lse, int32_t* n_valid, int32_t* dev_status,
                                    void* workspace, size_t workspace_bytes, void* stream);

/* Workspace bytes for ss_ce_forward_e4m3 (0 if the sizes are invalid or
 * d % 16 != 0); it also serves the build and the backward. */
SS_API size_t ss_workspace_bytes_e4m3(int64_t T, int32_t d, int32_t V, int32_t P);

/* The per-tensor e4m3 quantization ss_ce_forward_e4m3 applies, on its own:
 * dst[i] = code of src[i] * 2^-k (rounded to nearest even, saturating), with
 * 2^k as above written to scale[0] (device float).
 * In:  src [n] bf16, n % 8 == 0; scratch: 32 bytes of device memory (its
 *      first 8 bytes are cleared by the call). All pointers 16-byte aligned.
 * Out: dst [n] uint8 codes; scale [1] float32. */
SS_API ss_status ss_quantize_e4m3(const ss_bf16* src, int64_t n, uint8_t* dst, float* scale,
                                  void* scratch, void* stream);

/* Backward of the loss above for an upstream gradient g = grad_loss[0]
 * ("Learning Triton ... Softmax", section "Gradient": softmax minus one-hot):
 *   G     = (g / n_valid) * (softmax - onehot)  (0 when n_valid = 0);
 *   dx    = G @ W_C                      [T, d] bf16;
 *   dW    = dense [V, d] bf16: row C_j = (G^T @ x)_j, every other row +0.0
 *           (module docstring: the lm_head gradient spans the vocabulary).
 * Computed from the forward's workspace as dx = (g/n) r (.) (E' @ W_C) and
 * dW_C = (g/n) E'^T @ x'.
 * In:  grad_loss [1] float32 (device); candidates, vocab_pos as above; n_valid
 *      from ss_ce_forward; the workspace the forward used (it holds the x' rows).
 * Out: dx [T, d], dW [V, d] (fully written). Of the workspace the backward
 *      writes only the two GEMMs' tile counters (each GEMM hands its output
 *      tiles to CTA pairs through one; dX resets dW's and dW resets dX's), so
 *      the backward may be repeated (for another grad_loss) after one forward;
 *      as with every call, one workspace serves one stream at a time. */
SS_API ss_status ss_ce_backward(const float* grad_loss, const int32_t* candidates,
                         const int32_t* vocab_pos, const int32_t* n_valid, int64_t T,
                         int32_t d, int32_t V, int32_t P, ss_bf16* dx, ss_bf16* dW,
                         int32_t* dev_status, void* workspace, size_t workspace_bytes,
                         void* stream);

/* Human-readable name of a status code (static storage). */
SS_API const char* ss_status_string(int32_t status);

/* Text of the last CUDA runtime error seen by this thread ("" if none). */
SS_API const char* ss_last_cuda_error(void);

/* Library version, major * 10000 + minor * 100 + patch. */
SS_API int32_t ss_version(void);

/* Where each token's prefix target sits in C (sampled_softmax.py: module
 * docstring, CandidateBuilder.build and the SampledLoss field prefix_pos).
 * For token i with a valid target t_i the prefix target is
 * p_i = prefix_table[t_i]; prefix_pos[i] = vocab_pos[p_i] when p_i is a class
 * of C, and -1 otherwise: when p_i is a class outside C (that token then has
 * no prefix target, and prefix targets never add classes to C), when
 * p_i = -1 ("no prefix"), and for an ignored token (t_i = -1). The caller's
 * loss reads -1 as a no-op.
 * In:  prefix_table [V] int32, entries in [-1, V); targets [T] and vocab_pos
 *      [V] of the same microbatch as given to / written by ss_build_candidates.
 * Out: prefix_pos [T] int32.
 * A table entry outside [-1, V) or a target outside [-1, V) gives -1 for that
 * token and sets dev_status[8] = SS_ERR_BAD_INDEX (first error wins) with
 * dev_status[9] = 2 (table entry) or 3 (target). Needs no workspace. */
SS_API ss_status ss_prefix_positions(const int32_t* prefix_table, const int32_t* targets,
                                     const int32_t* vocab_pos, int64_t T, int32_t V,
                                     int32_t* prefix_pos, int32_t* dev_status, void* stream);

/* Self-test of the failure path every pipeline wait in the kernels shares
 * (the pages have no counterpart). Each wait on a TMA / MMA barrier is
 * bounded: after 2 s without progress the waiting warp raises its CTA's abort
 * flag, records SS_ERR_KERNEL_TIMEOUT in dev_status[8] (first error wins,
 * detail in [9]) and its kernel returns, so a stalled pipeline leaves an
 * error status and a usable context instead of a hung GPU. This call
 * launches one CTA whose first warp waits on a barrier that nothing
 * completes; its second warp starts a like wait 0.25 s later and must leave
 * through the abort flag. Afterwards, once the stream reaches it (about 2 s):
 *   dev_status[8]  = SS_ERR_KERNEL_TIMEOUT if [8] was 0 before
 *   dev_status[9]  = 107 (the self-test's kernel id)
 *   dev_status[10] = 1 if the second warp left through the abort flag
 *   dev_status[11] = the first warp's wait in whole milliseconds
 * Returns SS_OK once the kernel is enqueued. Occupies one SM for ~2 s. */
SS_API ss_status ss_selftest_wait_limit(int32_t* dev_status, void* stream);

/* Kernel timing for diagnostics. While enabled, each kernel launch the library
 * makes is bracketed by two CUDA events recorded on its stream (a pool of
 * 8192 launches, created by the first enabling call so that none is created
 * inside a timed region; later launches go untimed); enable = 2 brackets only
 * the tensor-core GEMM launches (fewer events in a timed loop), 1 every
 * launch, 0 none. An event between two launches also ends the overlap the
 * programmatic launch allows there. ss_timing_query synchronises on the
 * recorded events and returns, for the i-th distinct kernel name, its launch
 * count and total milliseconds. Not thread-safe; for benchmarks. */
SS_API ss_status ss_timing_enable(int32_t enable);
SS_API ss_status ss_timing_reset(void);
SS_API int32_t ss_timing_count(void);
SS_API ss_status ss_timing_query(int32_t i, char* name, int32_t name_len, int32_t* launches,
                          double* total_ms);

#ifdef __cplusplus
}
#endif

#endif /* SAMPLED_CE_H */
