// ce_gemm.cu -- the three dense contractions of the sampled-softmax CE head on
// the sm_100a tensor cores (tcgen05.mma, accumulators in TMEM, operands staged
// by TMA with 128-byte swizzle, no multicast):
//
//   forward : z[T,P]    = x[T,d] . W_C[P,d]^T     epilogue: E = exp(z - ref)
//   dX      : dx[T,d]   = r (.) (E'[T,P] . W_C)   epilogue: per-row scale
//   dW      : dW_C[P,d] = E'^T . x'[T,d]          epilogue: row scatter into dW[V,d]
//
// sampled_softmax.py (module docstring, "What"/"Why") counts them as the
// logits GEMM with its CE pass, and the pair of gradient GEMMs.
//
// The forward never stores the logits. Each row i has a reference logit ref_i
// computed beforehand (the logit of its target class), and the epilogue
// stores E = exp(z - ref_i) in bf16 together with, per row and per 256-column
// tile, the fp32 sum of those exponentials. With S_i the row's total,
//   lse_i = ref_i + log S_i,   softmax_ij = E_ij / S_i,
// ("Learning Triton One Kernel at a Time: Softmax": max-shifted softmax and
// the tile-wise sum of its "Online Softmax" section, with the target logit as
// the shift). Because loss_i = lse_i - z_target >= max_j z_ij - z_target, E
// can only grow large on a row whose loss is large; rows whose S_i reaches
// 2^64 (loss >= 44 nats) are recomputed exactly with the row maximum as the
// shift (ce_kernels.cu).
// After the forward, the row pass writes E'_{i,t_i} = 1 - S_i at the target
// column, r_i = 1 / S_i and x'_i = r_i x_i, so that r_i E'_ij is exactly
// softmax_ij - [j == t_i] (section "Gradient") and the backward is two plain
// GEMMs with epilogue scales: dX = (g/n) r (.) (E' W_C), dW_C = (g/n) E'^T x'.
//
// Work unit: an output tile computed by a CTA pair (a cluster of two CTAs on
// one TPC, tcgen05 cta_group::2). Each CTA loads its own 128-row block(s) of A
// and its 128-column half of B; the pair's leader issues M=256, N=256, K=16
// MMAs that read both CTAs' shared memory and write 128 rows x 256 fp32
// columns into each CTA's TMEM.
//   forward : 256 x 256 tiles, one A block per CTA; two TMEM accumulators let
//             the epilogue of tile i overlap the MMAs of tile i+1 (12 K blocks
//             per tile: the epilogue is a large share of a tile's time).
//   dX, dW  : 512 x 256 tiles, two A blocks per CTA and two MMAs per K step
//             sharing the B operand, both accumulators for one tile. Per
//             multiply-add this loads 25% fewer operand bytes from L2 than a
//             256 x 256 tile: at full clock the operand stream from L2 to the
//             SMs (about 11 TB/s measured) bounds these GEMMs, not the tensor
//             cores. Their K loops are hundreds of blocks long, so a
//             single-buffered accumulator costs under 1%.
// Tiles go to CTA pairs dynamically: each pair starts on tile `cluster` and
// then takes the next index from a counter in global memory (atomicAdd by the
// leader's producer, which passes it to both CTAs' warps through a small ring
// in shared memory), so pairs that start late -- their SMs still held by a
// kernel on another stream, such as a gradient all-reduce -- take fewer
// tiles instead of ending the kernel late. Tiles are taken in n-fastest
// order, so the pairs running at once share the A stripe.
// Per CTA, persistent over tiles:
//   warp 0      TMA producer, ring of stages (A 128x64 per block + B 128x64
//               bf16, or 128x128 e4m3 codes): 6 x 32 KB in the forward, 5 in
//               the e4m3 forward, 4 x 48 KB in dX and dW
//   warp 1      TMEM owner (2 x 256 columns); in the leader, the MMA issuer
//               (kind::f16, or kind::f8f6f4 with K=32 for the e4m3 forward)
//   warps 2..   epilogue: 8 warps in the forwards (two per TMEM lane quarter,
//               each over half of a tile's columns), 4 in dX and dW:
//               TMEM -> registers -> math -> global (forward: through swizzled
//               shared-memory boxes and TMA stores; dX, dW: 16-byte stores)
#include "sm100.cuh"
#include "ce_gemm.h"
#include "ss_internal.h"
#include "sampled_ce.h"

namespace ssb {

constexpr int BM = 128;          // rows per CTA (256 per pair)
constexpr int BN = 256;          // output columns per tile
constexpr int BNH = BN / 2;      // B columns held by each CTA of the pair
constexpr int BK = 64;
constexpr int A_STAGE = BM * BK * 2;   // 16 KB
constexpr int B_STAGE = BNH * BK * 2;  // 16 KB
constexpr int EPI_BUF = 32 * 64 * 2;  // one 32-row x 64-column bf16 box (4 KB)
constexpr int BAR_BYTES = 256;
// Slots of the tile-index ring. A slot is rewritten SCHED tiles after it was
// written, and by then every warp of the pair has read it: when the leader's
// producer starts tile s, the MMA warp has finished K block s * num_kb - 1 -
// STAGES (the stage it reloads), so it works on tile >= s - ceil(STAGES /
// num_kb) and the epilogue warps of both CTAs, which released that tile's
// accumulator ACC tiles earlier, have read the slot of tile s - ceil(STAGES /
// num_kb) - ACC - 1 or later; the peer's producer has loaded as far as the MMA
// warp has computed. So SCHED >= ceil(STAGES / num_kb) + ACC + 1, at most
// 7 + 2 + 1 here, is enough.
constexpr int SCHED = 12;
constexpr uint32_t TMEM_COLS = 2 * BN;
constexpr float LOG2E = 1.4426950408889634f;

// Per kind: operand majors, the E store path, pipeline stages and epilogue
// warps. The forward stores the 2.4 GB E stream through staging boxes and
// TMA bulk stores (1.47 ms against 1.89 ms with 16-byte register stores,
// measured); the boxes cost one operand stage. Its epilogue -- TMEM loads, an
// exponential per element, packing, staging and stores -- is busy for most of
// the kernel, stalled on dependency latency with one warp per scheduler: both
// forwards run two warps per TMEM lane quarter, each over half of the tile's
// columns (bf16: 3% faster with one staging box per warp, measured; two boxes
// per warp and one stage fewer gained nothing; e4m3, whose MMAs take half as
// long: 8% faster). dX and dW (hundreds of K blocks per
// tile) store little, from registers; their 48 KB stages (two A blocks) fit
// four times, 192 KB in flight per SM as with seven 32 KB stages.
// What the kernel computes: the forward (logits and E), dX, or dW_C with its scatter.
enum Role { ROLE_FWD = 0, ROLE_DX = 1, ROLE_DW = 2 };

template <int KIND>
struct Op;
template <>
struct Op<KIND_FWD> {  // A = x (K-major), B = W_C (K-major)
  static constexpr int ROLE = ROLE_FWD, A_MN = 0, B_MN = 0, TMA_STORE = 1, STAGES = 6,
                       EPI_WARPS = 8, AB = 1, EPI_BUFS = 1;
};
template <>
struct Op<KIND_FWD8> {  // A = x_q, B = W_C,q (e4m3, K-major; 128 per K block)
  static constexpr int ROLE = ROLE_FWD, A_MN = 0, B_MN = 0, TMA_STORE = 1, STAGES = 5,
                       EPI_WARPS = 8, AB = 1, EPI_BUFS = 2;
};
template <>
struct Op<KIND_DX> {  // A = E' (K-major), B = W_C viewed [K=P][N=d] (MN-major)
  static constexpr int ROLE = ROLE_DX, A_MN = 0, B_MN = 1, TMA_STORE = 0, STAGES = 4,
                       EPI_WARPS = 4, AB = 2, EPI_BUFS = 0;
};
template <>
struct Op<KIND_DW> {  // A = E' viewed [K=T][M=P] (MN-major), B = x' viewed [K=T][N=d] (MN-major)
  static constexpr int ROLE = ROLE_DW, A_MN = 1, B_MN = 1, TMA_STORE = 0, STAGES = 4,
                       EPI_WARPS = 4, AB = 2, EPI_BUFS = 0;
};
template <>
struct Op<KIND_DX1> {  // dX on 256-row tiles: 7 stages of 32 KB, two accumulators
  static constexpr int ROLE = ROLE_DX, A_MN = 0, B_MN = 1, TMA_STORE = 0, STAGES = 7,
                       EPI_WARPS = 4, AB = 1, EPI_BUFS = 0;
};
template <>
struct Op<KIND_DW1> {  // dW on 256-row tiles
  static constexpr int ROLE = ROLE_DW, A_MN = 1, B_MN = 1, TMA_STORE = 0, STAGES = 7,
                       EPI_WARPS = 4, AB = 1, EPI_BUFS = 0;
};

// Bytes of one pipeline stage: AB blocks of 128 A rows, and the CTA's half of B.
template <int KIND>
constexpr int stage_bytes() {
  return Op<KIND>::AB * A_STAGE + B_STAGE;
}
// Accumulator buffers in TMEM (2 x 256 columns): two tiles in flight when a
// tile takes one 256-column accumulator, one tile when it takes both.
template <int KIND>
constexpr int acc_bufs() {
  return Op<KIND>::AB == 1 ? 2 : 1;
}

static_assert(!Op<KIND_DX>::TMA_STORE && !Op<KIND_DW>::TMA_STORE && !Op<KIND_DX1>::TMA_STORE &&
                  !Op<KIND_DW1>::TMA_STORE,
              "only the forwards stage E for TMA stores");
static_assert(Op<KIND_FWD>::EPI_WARPS / 4 == kFwdSumsPerTileBf16 &&
                  Op<KIND_FWD8>::EPI_WARPS / 4 == kFwdSumsPerTileE4m3,
              "row sums per tile");

// warp 0 producer, warp 1 TMEM owner / MMA issuer, then the epilogue warps
template <int KIND>
constexpr int num_threads() {
  return 64 + 32 * Op<KIND>::EPI_WARPS;
}
template <int KIND>
constexpr int epi_bytes() {
  return Op<KIND>::TMA_STORE ? Op<KIND>::EPI_WARPS * Op<KIND>::EPI_BUFS * EPI_BUF : 0;
}
template <int KIND>
constexpr int smem_bytes() {
  return 1024 + Op<KIND>::STAGES * stage_bytes<KIND>() + epi_bytes<KIND>() + BAR_BYTES;
}
// barriers (full, empty per stage; tfull, tempty), the ring's slots, the TMEM
// address and the abort flag
template <int KIND>
constexpr int bar_bytes_used() {
  return (2 * Op<KIND>::STAGES + 4 + SCHED) * 8 + 8;
}
static_assert(bar_bytes_used<KIND_FWD>() <= BAR_BYTES && bar_bytes_used<KIND_FWD8>() <= BAR_BYTES &&
                  bar_bytes_used<KIND_DX>() <= BAR_BYTES && bar_bytes_used<KIND_DW>() <= BAR_BYTES &&
                  bar_bytes_used<KIND_DX1>() <= BAR_BYTES && bar_bytes_used<KIND_DW1>() <= BAR_BYTES,
              "barrier region");
static_assert(smem_bytes<KIND_FWD>() <= 232448 && smem_bytes<KIND_FWD8>() <= 232448 &&
                  smem_bytes<KIND_DX>() <= 232448 && smem_bytes<KIND_DW>() <= 232448 &&
                  smem_bytes<KIND_DX1>() <= 232448 && smem_bytes<KIND_DW1>() <= 232448,
              "shared memory budget");

// One lane's 64 values of a chunk, as bf16, into row `lane` of a 32 x 64
// staging box with the 128-byte swizzle of the E store's tensor map.
SS_DEV void stage_box(uint32_t row_addr, int lane, const float (&v)[64]) {
#pragma unroll
  for (int cc = 0; cc < 8; ++cc) {
    st_shared_v4(row_addr + ((cc ^ (lane & 7)) << 4), pack_bf16x2(v[cc * 8 + 0], v[cc * 8 + 1]),
                 pack_bf16x2(v[cc * 8 + 2], v[cc * 8 + 3]), pack_bf16x2(v[cc * 8 + 4], v[cc * 8 + 5]),
                 pack_bf16x2(v[cc * 8 + 6], v[cc * 8 + 7]));
  }
}

SS_DEV void raise_abort(volatile int* abort_flag, int32_t* status, int kind) {
  *abort_flag = 1;
  if (status != nullptr) {
    if (atomicCAS(status, 0, (int32_t)SS_ERR_KERNEL_TIMEOUT) == 0) status[1] = 100 + kind;
  }
}

// Warp-uniform bounded wait.
SS_DEV bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag, int32_t* status,
                      int kind) {
  bool ok = mbar_wait(bar, parity, abort_flag);
  ok = __all_sync(0xffffffffu, ok);
  if (!ok) raise_abort(abort_flag, status, kind);
  return ok;
}

// The tile-index ring. Slot `it % SCHED` holds {it + 1, tile}: the tile that
// follows a warp's `it`-th tile (an index >= the tile count ends the warp's
// loop). The leader's producer writes both CTAs' copies with plain 64-bit
// stores (the peer's through its shared::cluster address); the other warps
// of the pair (the leader's MMA warp, the peer's producer, the epilogue warps
// of both CTAs) poll their own copy until its tag is it + 1. The value is its
// own flag, so neither side needs a fence or a barrier, and the slot is not
// rewritten before every warp has read it (SCHED, above). A tag past it + 1
// would mean a warp fell behind that bound: it is reported, not used.
SS_DEV void ring_publish(volatile uint64_t* ring, int it, int tile) {
  if ((threadIdx.x & 31) == 0) {
    const int j = it % SCHED;
    const uint64_t v = ((uint64_t)((uint32_t)it + 1u) << 32) | (uint32_t)tile;
    ring[j] = v;
    st_shared_cluster_u64(mapa_shared(smem_u32((const void*)(ring + j)), 1), v);
  }
  __syncwarp();
}

SS_DEV bool ring_next(const volatile uint64_t* ring, int it, int* tile, volatile int* abort_flag,
                      int32_t* status, int kind) {
  const int j = it % SCHED;
  const uint32_t want = (uint32_t)it + 1u;
  uint64_t v = ring[j];
  bool ok = (uint32_t)(v >> 32) == want;
  if (!ok) {
    const unsigned long long t0 = globaltimer();
    for (uint32_t k = 1;; ++k) {
      v = ring[j];
      const uint32_t tag = (uint32_t)(v >> 32);
      if (tag == want) {
        ok = true;
        break;
      }
      if (tag > want) break;  // overwritten: cannot happen within the bound
      if ((k & 31u) == 0 && (*abort_flag || globaltimer() - t0 > kWaitLimitNs)) break;
    }
  }
  ok = __all_sync(0xffffffffu, ok);
  if (!ok) {
    raise_abort(abort_flag, status, kind);
    return false;
  }
  *tile = __shfl_sync(0xffffffffu, (int)(uint32_t)v, 0);
  return true;
}

// Self-test of the bounded wait above, on one CTA of two warps. Warp 0 waits
// on a barrier that nothing completes and, when the limit passes, raises the
// abort flag and records SS_ERR_KERNEL_TIMEOUT -- what a GEMM warp does when
// its pipeline stalls. Warp 1 begins its own wait on a second such barrier an
// eighth of the limit later, so it must leave through the flag before its
// own limit, as the other warps of a stalled GEMM do. status = dev_status + 8:
// [0] error, [1] detail (100 + 7), [2] 1 if warp 1 left through the flag,
// [3] warp 0's wait in milliseconds.
__global__ void __launch_bounds__(64, 1) k_wait_selftest(int32_t* status) {
  pdl_wait();
  pdl_trigger();
  __shared__ __align__(8) uint64_t bars[2];
  __shared__ int abort_word;
  volatile int* abort_flag = &abort_word;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (warp == 1) {
    const unsigned long long t = globaltimer();
    while (globaltimer() - t < kWaitLimitNs / 8) __nanosleep(1000);
  }
  const unsigned long long t0 = globaltimer();
  const bool ok = warp_wait(&bars[warp], 0u, abort_flag, status, 7);
  const unsigned long long waited = globaltimer() - t0;
  if (lane == 0) {
    if (warp == 0) status[3] = (int32_t)(waited / 1000000ull);
    if (warp == 1) status[2] = (!ok && waited < kWaitLimitNs) ? 1 : 0;
  }
}

cudaError_t launch_wait_selftest(int32_t* status, cudaStream_t s) {
  return launch_pdl(k_wait_selftest, dim3(1), dim3(64), 0, s, status);
}

template <int KIND>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(num_threads<KIND>(), 1)
    k_gemm(const __grid_constant__ CUtensorMap tma_a, const __grid_constant__ CUtensorMap tma_b,
           const __grid_constant__ CUtensorMap tma_c, const GemmArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  constexpr int STAGES = Op<KIND>::STAGES;
  constexpr int AB = Op<KIND>::AB;             // 128-row A blocks per CTA and tile
  constexpr int ACC = acc_bufs<KIND>();        // tiles whose accumulators fit in TMEM
  constexpr int STAGE = stage_bytes<KIND>();
  constexpr int TILE_ROWS = 2 * BM * AB;       // output rows of a pair's tile
  constexpr bool IS_FWD = KIND == KIND_FWD || KIND == KIND_FWD8;
  constexpr bool F8 = KIND == KIND_FWD8;
  constexpr int BKE = F8 ? 2 * BK : BK;  // K elements per 128-byte row of a stage
  uint8_t* epi_smem = smem + STAGES * STAGE;
  uint64_t* full = reinterpret_cast<uint64_t*>(epi_smem + epi_bytes<KIND>());
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  volatile uint64_t* ring = tempty + 2;  // [SCHED] tile-index ring
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(tempty + 2 + SCHED);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0 = the pair's leader
  const int cluster = blockIdx.x >> 1, num_clusters = gridDim.x >> 1;
  const int num_tiles = args.tiles_m * args.tiles_n;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);   // leader: one expect-tx arrival for both CTAs' bytes
      mbar_init(&empty[s], 1);  // one multicast commit from the leader's MMA
    }
    for (int a = 0; a < ACC; ++a) {
      mbar_init(&tfull[a], 1);   // one multicast commit per finished accumulator
      mbar_init(&tempty[a], 2 * Op<KIND>::EPI_WARPS);  // leader: epilogue warps of both CTAs
    }
    for (int j = 0; j < SCHED; ++j) ring[j] = 0;  // no tag yet
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {  // descriptors live in kernel parameter space
    tma_prefetch_desc(&tma_a);
    tma_prefetch_desc(&tma_b);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_holder, TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();  // barriers of both CTAs initialised, TMEM allocated
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  // set-up above overlaps the previous kernel's tail; global memory only from here
  pdl_wait();
  pdl_trigger();
  if (blockIdx.x == 0 && threadIdx.x == 0 && args.next_ctr != nullptr) *args.next_ctr = 0;

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer --
    // B (W_C, or x' in dW) is reused by every tile: keep it in L2
    const uint64_t keep_b = policy_evict_last();
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    // The leader fetches two tiles ahead: once the first loads of its it-th
    // tile are issued it publishes the following tile (fetched a tile
    // earlier, so the atomic's latency has passed) and fetches the one after
    // that. The peer's producer then finds its next tile published when it
    // needs it. A fetch left unpublished when the loop ends came after the
    // index that ended it, so it is past the last tile too.
    auto fetch = [&](int fallback) {
      int v = fallback;
      if (rank == 0 && lane == 0 && args.tile_ctr != nullptr)
        v = num_clusters + atomicAdd(args.tile_ctr, 1);
      return v;
    };
    int tile = cluster;
    int next = fetch(cluster + num_clusters);
    for (int it = 0; ok && tile < num_tiles; ++it) {
      int after = 0;
      // A block b of this CTA: rows m0 + b * 2 * BM .. + BM (the pair's
      // 256-row MMA b takes block b of both CTAs)
      const int m0 = (tile / args.tiles_n) * TILE_ROWS + (int)rank * BM;
      const int nh0 = (tile % args.tiles_n) * BN + (int)rank * BNH;
      for (int kb = 0; kb < args.num_kb; ++kb) {
        if (!warp_wait(&empty[stage], phase ^ 1u, abort_flag, args.status, KIND)) {
          ok = false;
          break;
        }
        if (lane == 0) {
          uint8_t* sa = smem + stage * STAGE;
          uint8_t* sb = sa + AB * A_STAGE;
          const int k0 = kb * BKE;
          // a TMA box must start on a 16-byte boundary of its inner dimension
          // (a failed check skips the loads; the pipeline then times out)
          const bool aligned = SS_CHECK((k0 * (F8 ? 1 : 2)) % 16 == 0, args.status, 9);
          if (aligned && rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * STAGE);
          if (aligned) {
            const uint32_t bar = mapa_shared(smem_u32(&full[stage]), 0);
#pragma unroll
            for (int b = 0; b < AB; ++b) {
              const int mb = m0 + b * 2 * BM;
              if (Op<KIND>::A_MN) {
                tma_load_2d_pair(sa + b * A_STAGE, &tma_a, bar, mb, k0);
                tma_load_2d_pair(sa + b * A_STAGE + 8192, &tma_a, bar, mb + 64, k0);
              } else {
                tma_load_2d_pair(sa + b * A_STAGE, &tma_a, bar, k0, mb);
              }
            }
            if (Op<KIND>::B_MN) {
              tma_load_2d_pair_hint(sb, &tma_b, bar, nh0, k0, keep_b);
              tma_load_2d_pair_hint(sb + 8192, &tma_b, bar, nh0 + 64, k0, keep_b);
            } else {
              tma_load_2d_pair_hint(sb, &tma_b, bar, k0, nh0, keep_b);
            }
          }
        }
        __syncwarp();
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
        if (kb == 0 && rank == 0) {  // after this tile's first loads are on their way
          next = __shfl_sync(0xffffffffu, next, 0);
          ring_publish(ring, it, next);
          after = fetch(next + num_clusters);
        }
      }
      if (!ok) break;
      if (rank == 0) {
        tile = next;
        next = after;
      } else if (!ring_next(ring, it, &tile, abort_flag, args.status, KIND)) {
        ok = false;
        break;
      }
    }
    // Wait until the last stages are released, so that no MMA-completion
    // arrival is still on its way to this CTA's barriers when it exits.
    for (int i = 0; ok && i < STAGES; ++i) {
      if (!warp_wait(&empty[stage], phase ^ 1u, abort_flag, args.status, KIND)) break;
      if (++stage == STAGES) {
        stage = 0;
        phase ^= 1u;
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------- MMA issuer (leader only) --
    if (rank == 0) {
      constexpr uint32_t IDESC =
          F8 ? idesc_e4m3(2 * BM, BN) : idesc_bf16(2 * BM, BN, Op<KIND>::A_MN, Op<KIND>::B_MN);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int tile = cluster;
      for (int it = 0; ok && tile < num_tiles; ++it) {
        const int acc = it % ACC;
        const uint32_t acc_phase = (it / ACC) & 1;
        if (!warp_wait(&tempty[acc], acc_phase ^ 1u, abort_flag, args.status, KIND)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * AB * BN;  // block b: + b * BN
        for (int kb = 0; kb < args.num_kb; ++kb) {
          if (!warp_wait(&full[stage], phase, abort_flag, args.status, KIND)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (lane == 0) {
            const uint32_t a_addr = smem_u32(smem + stage * STAGE);
            const uint32_t b_addr = a_addr + AB * A_STAGE;
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk) {
              const uint64_t bd = Op<KIND>::B_MN ? sdesc_sw128(b_addr + kk * 2048, 8192, 1024)
                                                 : sdesc_sw128(b_addr + kk * 32, 16, 1024);
#pragma unroll
              for (int b = 0; b < AB; ++b) {
                const uint32_t ab = a_addr + b * A_STAGE;
                const uint64_t ad = Op<KIND>::A_MN ? sdesc_sw128(ab + kk * 2048, 8192, 1024)
                                                   : sdesc_sw128(ab + kk * 32, 16, 1024);
                if (F8)  // K = 32 e4m3 per MMA: the same 32 bytes as 16 bf16
                  umma_f8_pair(d_tmem + b * BN, ad, bd, IDESC, (kb | kk) != 0 ? 1u : 0u);
                else
                  umma_bf16_pair(d_tmem + b * BN, ad, bd, IDESC, (kb | kk) != 0 ? 1u : 0u);
              }
            }
            umma_commit_pair(&empty[stage], 0x3);  // frees the stage in both CTAs
          }
          __syncwarp();
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        if (lane == 0) umma_commit_pair(&tfull[acc], 0x3);  // both halves of the tile ready
        __syncwarp();
        if (!ring_next(ring, it, &tile, abort_flag, args.status, KIND)) break;
      }
    }
  } else {
    // ----------------------------------------------------------- epilogue --
    constexpr int EW = Op<KIND>::EPI_WARPS;
    constexpr int HALVES = EW / 4;        // warps per TMEM lane quarter
    constexpr int CPW = BN / 64 / HALVES;  // 64-column chunks per warp and tile
    const int q = warp & 3;   // TMEM lane quarter this warp may access
    const int e = warp - 2;   // staging slot
    const int half = e / 4;   // which part of the tile's columns
    const int c_begin = half * CPW;
    uint32_t store_ctr = 0;
    // the forward's E is a write-once stream larger than L2: evict it first
    const uint64_t store_policy = IS_FWD ? policy_evict_first() : 0;
    // forward: log2(e) times the logits' scale (the operand scales for e4m3)
    const float zs = F8 ? LOG2E * __ldg(args.qscale + 2) : LOG2E;
    float scale = 1.f;  // dX / dW: g / n (0 when no row is valid)
    if (!IS_FWD) {
      const int nv = __ldg(args.n_valid);
      scale = nv > 0 ? __ldg(args.grad_loss) / (float)nv : 0.f;
    }
    if (Op<KIND>::ROLE == ROLE_DW && args.vocab_pos != nullptr) {
      // The rows of dW outside C are +0.0. The epilogue warps of every CTA
      // write them while the first tiles' MMAs run (they are disjoint from
      // the rows the tiles scatter). Each warp takes blocks of 32 classes.
      const int vpr = args.N / 8;
      const int64_t gw = (int64_t)blockIdx.x * EW + e, nw = (int64_t)gridDim.x * EW;
      uint4* dW4 = reinterpret_cast<uint4*>(args.dW);
      for (int64_t base = gw * 32; base < args.V; base += nw * 32) {
        const int64_t r = base + lane;
        const bool zero_row = r < args.V && __ldg(args.vocab_pos + r) < 0;
        unsigned m = __ballot_sync(0xffffffffu, zero_row);
        while (m) {
          const int k = __ffs(m) - 1;
          m &= m - 1;
          uint4* dst = dW4 + (base + k) * vpr;
          for (int v = lane; v < vpr; v += 32) __stcs(dst + v, make_uint4(0, 0, 0, 0));
        }
      }
    }
    int tile = cluster;
    for (int it = 0; tile < num_tiles; ++it) {
      const int acc = it % ACC;
      const uint32_t acc_phase = (it / ACC) & 1;
      const int m_blk = tile / args.tiles_n, n_blk = tile % args.tiles_n;
      const int n0 = n_blk * BN;
      // this lane's row in A block b is row0 + b * 2 * BM
      const int row0 = m_blk * TILE_ROWS + (int)rank * BM + q * 32 + lane;

      // per-row values, loaded before the accumulator is ready
      // forward: ref_i * log2(e), and whether E is stored (0 on ignored rows),
      // for A blocks 0 and 1
      float ref2_0 = 0.f, ref2_1 = 0.f;
      bool keep0 = true, keep1 = true;
      // dX: (g / n) * r_i and dW: the row's class id, for A blocks 0 and 1
      float rs0 = scale, rs1 = scale;
      int32_t cls0 = -1, cls1 = -1;
      if (IS_FWD && row0 < args.M) {
        ref2_0 = __ldg(args.ref + row0) * LOG2E;
        keep0 = __ldg(args.tpos + row0) >= 0;
      }
      if (IS_FWD && AB > 1 && row0 + 2 * BM < args.M) {
        ref2_1 = __ldg(args.ref + row0 + 2 * BM) * LOG2E;
        keep1 = __ldg(args.tpos + row0 + 2 * BM) >= 0;
      }
      if (Op<KIND>::ROLE == ROLE_DX) {
        rs0 = row0 < args.M ? scale * __ldg(args.rscale + row0) : 0.f;
        if (AB > 1) rs1 = row0 + 2 * BM < args.M ? scale * __ldg(args.rscale + row0 + 2 * BM) : 0.f;
      }
      if (Op<KIND>::ROLE == ROLE_DW) {
        if (row0 < args.M) cls0 = __ldg(args.cand + row0);
        if (AB > 1 && row0 + 2 * BM < args.M) cls1 = __ldg(args.cand + row0 + 2 * BM);
      }

      if (!warp_wait(&tfull[acc], acc_phase, abort_flag, args.status, KIND)) break;
      tc_fence_after();

      const int n_chunks = min(BN / 64, (args.N - n0 + 63) / 64);  // with valid columns
      const int c_end = min(c_begin + CPW, n_chunks);
      if (c_begin >= c_end) {  // no valid column of this tile for this warp
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&tempty[acc]), 0));
      }

#pragma unroll 1
      for (int b = 0; b < AB; ++b) {
        const int row = row0 + b * 2 * BM;
        const bool row_ok = row < args.M;
        const float rs = b == 0 ? rs0 : rs1;
        const int32_t cl = b == 0 ? cls0 : cls1;
        const float ref2 = b == 0 ? ref2_0 : ref2_1;
        const bool keep = b == 0 ? keep0 : keep1;
        float s_tile = 0.f;
        const uint32_t t_row =
            tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)((acc * AB + b) * BN);
        if (!SS_CHECK((acc * AB + b + 1) * BN <= (int)TMEM_COLS, args.status, 8)) continue;
        for (int c = c_begin; c < c_end; ++c) {
          const int col0 = n0 + c * 64;
          uint32_t r0[32], r1[32];
          tmem_ld32(t_row + c * 64, r0);
          tmem_ld32(t_row + c * 64 + 32, r1);
          tmem_wait_ld();
          if (b == AB - 1 && c == c_end - 1) {
            // all TMEM reads of this accumulator are done: hand it back to the leader
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&tempty[acc]), 0));
          }
          float v[64];
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            v[j] = __uint_as_float(r0[j]);
            v[32 + j] = __uint_as_float(r1[j]);
          }

          if (IS_FWD) {
            // E = exp(z - ref) and its row sum over the tile's valid columns
            const int nvalid = min(64, args.N - col0);
            float sp[8];  // independent partial sums (short dependency chains)
#pragma unroll
            for (int u = 0; u < 8; ++u) sp[u] = 0.f;
            if (nvalid == 64) {
#pragma unroll
              for (int j = 0; j < 64; ++j) {
                v[j] = ex2_approx(fmaf(v[j], zs, -ref2));
                sp[j & 7] += v[j];
              }
            } else {
#pragma unroll
              for (int j = 0; j < 64; ++j) {
                v[j] = j < nvalid ? ex2_approx(fmaf(v[j], zs, -ref2)) : 0.f;
                sp[j & 7] += v[j];
              }
            }
            s_tile += ((sp[0] + sp[1]) + (sp[2] + sp[3])) + ((sp[4] + sp[5]) + (sp[6] + sp[7]));
            if (!keep) {
#pragma unroll
              for (int j = 0; j < 64; ++j) v[j] = 0.f;
            }
          } else if (Op<KIND>::ROLE == ROLE_DX) {
#pragma unroll
            for (int j = 0; j < 64; ++j) v[j] *= rs;
          } else {
#pragma unroll
            for (int j = 0; j < 64; ++j) v[j] *= scale;
          }

          if (Op<KIND>::TMA_STORE) {
            // bf16 tile -> swizzled staging box -> TMA store
            constexpr int NB = Op<KIND>::EPI_BUFS > 0 ? Op<KIND>::EPI_BUFS : 1;
            const uint32_t lane_off = lane * 128;
            const int box_row = row - lane;  // first row of this warp's 32-row boxes
            if (NB >= CPW) {
              // a box per chunk of this warp's columns: one async-proxy fence and
              // one bulk group for all of them (e4m3 forward: 2% faster, measured)
              const int slot = c - c_begin;
              uint8_t* buf = epi_smem + (e * NB + slot) * EPI_BUF;
              if (slot == 0) {  // the previous tile's stores have read this warp's boxes
                if (lane == 0) bulk_wait_read<0>();
                __syncwarp();
              }
              stage_box(smem_u32(buf) + lane_off, lane, v);
              if (c == c_end - 1) {
                fence_async_smem();
                __syncwarp();
                if (lane == 0 && box_row < args.M) {
                  for (int sl = 0; sl <= slot; ++sl)
                    tma_store_2d_hint(&tma_c, epi_smem + (e * NB + sl) * EPI_BUF,
                                      n0 + (c_begin + sl) * 64, box_row, store_policy);
                  bulk_commit();
                }
              }
            } else {
              // a ring of NB boxes: fence and store each chunk as it is staged
              uint8_t* buf = epi_smem + (e * NB + (int)(store_ctr % NB)) * EPI_BUF;
              if (lane == 0) bulk_wait_read<NB - 1>();  // this buffer's last store has read it
              __syncwarp();
              stage_box(smem_u32(buf) + lane_off, lane, v);
              fence_async_smem();
              __syncwarp();
              if (lane == 0 && box_row < args.M) {
                tma_store_2d_hint(&tma_c, buf, col0, box_row, store_policy);
                bulk_commit();
              }
            }
            ++store_ctr;
          } else if (Op<KIND>::ROLE != ROLE_DW) {
            // bf16 row segment straight from registers (16-byte stores)
            if (row_ok) {
              uint4* dst = reinterpret_cast<uint4*>(args.out + (size_t)row * args.ld_out + col0);
#pragma unroll
              for (int cc = 0; cc < 8; ++cc) {
                if (col0 + cc * 8 < args.N) {
                  const uint4 w = make_uint4(pack_bf16x2(v[cc * 8 + 0], v[cc * 8 + 1]),
                                             pack_bf16x2(v[cc * 8 + 2], v[cc * 8 + 3]),
                                             pack_bf16x2(v[cc * 8 + 4], v[cc * 8 + 5]),
                                             pack_bf16x2(v[cc * 8 + 6], v[cc * 8 + 7]));
                  if (IS_FWD)
                    __stcs(dst + cc, w);  // E is a write-once stream: do not keep it in L2
                  else
                    dst[cc] = w;
                }
              }
            }
          } else {  // KIND_DW: row `row` of dW_C goes to row cand[row] of dW
            if (row_ok && !(cl >= 0 && cl < args.V)) (void)SS_CHECK(false, args.status, 7);
            if (row_ok && cl >= 0 && cl < args.V) {
              uint4* dst = reinterpret_cast<uint4*>(args.dW + (size_t)cl * args.N + col0);
#pragma unroll
              for (int cc = 0; cc < 8; ++cc) {
                if (col0 + cc * 8 < args.N) {
                  uint4 w;
                  w.x = pack_bf16x2(v[cc * 8 + 0], v[cc * 8 + 1]);
                  w.y = pack_bf16x2(v[cc * 8 + 2], v[cc * 8 + 3]);
                  w.z = pack_bf16x2(v[cc * 8 + 4], v[cc * 8 + 5]);
                  w.w = pack_bf16x2(v[cc * 8 + 6], v[cc * 8 + 7]);
                  dst[cc] = w;
                }
              }
            }
          }
        }
        if (IS_FWD && row_ok) args.rowsum[(size_t)(n_blk * HALVES + half) * args.M + row] = s_tile;
      }
      if (!ring_next(ring, it, &tile, abort_flag, args.status, KIND)) break;
    }
    if (lane == 0) bulk_wait<0>();
    __syncwarp();
  }

  __syncthreads();
  if (*abort_flag) {
    // Let copies and MMAs already in flight land before TMEM is released.
    if (threadIdx.x == 0) {
      const unsigned long long t0 = globaltimer();
      while (globaltimer() - t0 < 2000000ull) __nanosleep(20000);
    }
    __syncthreads();
  }
  tc_fence_before();
  cluster_sync();  // neither CTA touches the other's memory or TMEM any more
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

int gemm_tile_rows(int kind) {
  switch (kind) {
    case KIND_FWD: return 2 * BM * Op<KIND_FWD>::AB;
    case KIND_FWD8: return 2 * BM * Op<KIND_FWD8>::AB;
    case KIND_DX: return 2 * BM * Op<KIND_DX>::AB;
    case KIND_DX1: return 2 * BM * Op<KIND_DX1>::AB;
    case KIND_DW1: return 2 * BM * Op<KIND_DW1>::AB;
    default: return 2 * BM * Op<KIND_DW>::AB;
  }
}

int gemm_smem_bytes(int kind) {
  switch (kind) {
    case KIND_FWD: return smem_bytes<KIND_FWD>();
    case KIND_FWD8: return smem_bytes<KIND_FWD8>();
    case KIND_DX: return smem_bytes<KIND_DX>();
    case KIND_DX1: return smem_bytes<KIND_DX1>();
    case KIND_DW1: return smem_bytes<KIND_DW1>();
    default: return smem_bytes<KIND_DW>();
  }
}

const void* gemm_kernel_ptr(int kind) {
  switch (kind) {
    case KIND_FWD: return reinterpret_cast<const void*>(&k_gemm<KIND_FWD>);
    case KIND_FWD8: return reinterpret_cast<const void*>(&k_gemm<KIND_FWD8>);
    case KIND_DX: return reinterpret_cast<const void*>(&k_gemm<KIND_DX>);
    case KIND_DX1: return reinterpret_cast<const void*>(&k_gemm<KIND_DX1>);
    case KIND_DW1: return reinterpret_cast<const void*>(&k_gemm<KIND_DW1>);
    default: return reinterpret_cast<const void*>(&k_gemm<KIND_DW>);
  }
}

// How many CTA pairs of this kernel can be resident at once on the device.
int gemm_threads(int kind) {
  switch (kind) {
    case KIND_FWD: return num_threads<KIND_FWD>();
    case KIND_FWD8: return num_threads<KIND_FWD8>();
    case KIND_DX: return num_threads<KIND_DX>();
    case KIND_DX1: return num_threads<KIND_DX1>();
    case KIND_DW1: return num_threads<KIND_DW1>();
    default: return num_threads<KIND_DW>();
  }
}

int gemm_max_pairs(int kind, int sms) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * (sms / 2));
  cfg.blockDim = dim3(gemm_threads(kind));
  cfg.dynamicSmemBytes = gemm_smem_bytes(kind);
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeClusterDimension;
  attr.val.clusterDim.x = 2;
  attr.val.clusterDim.y = 1;
  attr.val.clusterDim.z = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, gemm_kernel_ptr(kind), &cfg) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    n = sms / 2;
  }
  return n;
}

cudaError_t launch_gemm(int kind, const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& c,
                        const GemmArgs& args, int pairs, cudaStream_t s) {
  dim3 g(2 * pairs), blk(gemm_threads(kind));
  switch (kind) {
    case KIND_FWD: return launch_pdl(k_gemm<KIND_FWD>, g, blk, smem_bytes<KIND_FWD>(), s, a, b, c, args);
    case KIND_FWD8:
      return launch_pdl(k_gemm<KIND_FWD8>, g, blk, smem_bytes<KIND_FWD8>(), s, a, b, c, args);
    case KIND_DX: return launch_pdl(k_gemm<KIND_DX>, g, blk, smem_bytes<KIND_DX>(), s, a, b, c, args);
    case KIND_DX1:
      return launch_pdl(k_gemm<KIND_DX1>, g, blk, smem_bytes<KIND_DX1>(), s, a, b, c, args);
    case KIND_DW1:
      return launch_pdl(k_gemm<KIND_DW1>, g, blk, smem_bytes<KIND_DW1>(), s, a, b, c, args);
    default: return launch_pdl(k_gemm<KIND_DW>, g, blk, smem_bytes<KIND_DW>(), s, a, b, c, args);
  }
}

}  // namespace ssb
