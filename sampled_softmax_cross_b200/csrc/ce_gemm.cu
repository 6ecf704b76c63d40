// ce_gemm.cu -- the three dense contractions of the sampled-softmax CE head on
// the sm_100a tensor cores (tcgen05.mma, accumulators in TMEM, operands staged
// by TMA with 128-byte swizzle, no multicast):
//
//   forward : z[T,P]   = x[T,d] . W_C[P,d]^T   + online-softmax CE epilogue
//   dX      : dx[T,d]  = G[T,P] . W_C[P,d]
//   dW      : dW_C[P,d]= G[T,P]^T . x[T,d]      + row scatter into dW[V,d]
//
// sampled_softmax.py (module docstring, "What"/"Why") names these as the
// logits GEMM, the CE pass and the "two gradient GEMMs". The epilogue of the
// forward keeps, per row and per 256-column tile, the running maximum and the
// sum of exp(z - max) ("Learning Triton One Kernel at a Time: Softmax",
// section "Online Softmax": the tile version adds the tile's sum, rescaled,
// to the running sum), picks the fp32 logit of the target column, and stores
// the bf16 logits for the backward.
//
// One persistent CTA per SM, 192 threads:
//   warp 0      TMA producer (4-stage shared-memory ring, 48 KB per stage)
//   warp 1      MMA issuer (one thread) and TMEM owner (2 x 256 fp32 columns)
//   warps 2..5  epilogue: TMEM -> registers -> math -> shared -> TMA store
// Tiles are 128 x 256 with K blocks of 64; the two TMEM accumulators let the
// epilogue of tile i overlap the MMAs of tile i+1.
#include "sm100.cuh"
#include "ss_internal.h"

namespace ssb {

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
constexpr int A_STAGE = BM * BK * 2;  // 16 KB
constexpr int B_STAGE = BN * BK * 2;  // 32 KB
constexpr int STAGE_BYTES = A_STAGE + B_STAGE;
constexpr int EPI_BUF = 32 * 64 * 2;  // one 32-row x 64-column bf16 box (4 KB)
constexpr int EPI_BYTES = 4 * 2 * EPI_BUF;
constexpr int BAR_BYTES = 256;
constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + EPI_BYTES + BAR_BYTES;
constexpr uint32_t TMEM_COLS = 2 * BN;
constexpr int NUM_THREADS = 192;
constexpr float LOG2E = 1.4426950408889634f;

static_assert(SMEM_BYTES <= 232448, "shared memory budget");

template <int KIND>
struct Op;
template <>
struct Op<KIND_FWD> {  // A = x (K-major), B = W_C (K-major)
  static constexpr int A_MN = 0, B_MN = 0;
};
template <>
struct Op<KIND_DX> {  // A = G (K-major), B = W_C viewed [K=P][N=d] (MN-major)
  static constexpr int A_MN = 0, B_MN = 1;
};
template <>
struct Op<KIND_DW> {  // A = G viewed [K=T][M=P] (MN-major), B = x viewed [K=T][N=d] (MN-major)
  static constexpr int A_MN = 1, B_MN = 1;
};

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

template <int KIND>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    k_gemm(const __grid_constant__ CUtensorMap tma_a, const __grid_constant__ CUtensorMap tma_b,
           const __grid_constant__ CUtensorMap tma_c, const GemmArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* epi_smem = smem + STAGES * STAGE_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(epi_smem + EPI_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(tempty + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int num_tiles = args.tiles_m * args.tiles_n;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 4);  // one arrival per epilogue warp
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer --
    if (lane == 0) {
      tma_prefetch_desc(&tma_a);
      tma_prefetch_desc(&tma_b);
    }
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
      const int m0 = (tile / args.tiles_n) * BM, n0 = (tile % args.tiles_n) * BN;
      for (int kb = 0; kb < args.num_kb; ++kb) {
        if (!warp_wait(&empty[stage], phase ^ 1u, abort_flag, args.status, KIND)) {
          ok = false;
          break;
        }
        if (lane == 0) {
          uint8_t* sa = smem + stage * STAGE_BYTES;
          uint8_t* sb = sa + A_STAGE;
          const int k0 = kb * BK;
          mbar_arrive_expect_tx(&full[stage], STAGE_BYTES);
          if (Op<KIND>::A_MN) {
            tma_load_2d(sa, &tma_a, &full[stage], m0, k0);
            tma_load_2d(sa + 8192, &tma_a, &full[stage], m0 + 64, k0);
          } else {
            tma_load_2d(sa, &tma_a, &full[stage], k0, m0);
          }
          if (Op<KIND>::B_MN) {
#pragma unroll
            for (int i = 0; i < 4; ++i) tma_load_2d(sb + i * 8192, &tma_b, &full[stage], n0 + 64 * i, k0);
          } else {
            tma_load_2d(sb, &tma_b, &full[stage], k0, n0);
          }
        }
        __syncwarp();
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
  } else if (warp == 1) {
    // --------------------------------------------------------- MMA issuer --
    constexpr uint32_t IDESC = idesc_bf16(BM, BN, Op<KIND>::A_MN, Op<KIND>::B_MN);
    int stage = 0;
    uint32_t phase = 0;
    int it = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x, ++it) {
      const int acc = it & 1;
      const uint32_t acc_phase = (it >> 1) & 1;
      if (!warp_wait(&tempty[acc], acc_phase ^ 1u, abort_flag, args.status, KIND)) break;
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + acc * BN;
      for (int kb = 0; kb < args.num_kb; ++kb) {
        if (!warp_wait(&full[stage], phase, abort_flag, args.status, KIND)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (lane == 0) {
          const uint32_t a_addr = smem_u32(smem + stage * STAGE_BYTES);
          const uint32_t b_addr = a_addr + A_STAGE;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t ad = Op<KIND>::A_MN ? sdesc_sw128(a_addr + kk * 2048, 8192, 1024)
                                               : sdesc_sw128(a_addr + kk * 32, 16, 1024);
            const uint64_t bd = Op<KIND>::B_MN ? sdesc_sw128(b_addr + kk * 2048, 8192, 1024)
                                               : sdesc_sw128(b_addr + kk * 32, 16, 1024);
            umma_bf16(d_tmem, ad, bd, IDESC, (kb | kk) != 0 ? 1u : 0u);
          }
          umma_commit(&empty[stage]);  // frees the stage once these MMAs have read it
        }
        __syncwarp();
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) break;
      if (lane == 0) umma_commit(&tfull[acc]);  // accumulator ready for the epilogue
      __syncwarp();
    }
  } else {
    // ----------------------------------------------------------- epilogue --
    const int q = warp & 3;   // TMEM lane quarter this warp may access
    const int e = warp - 2;   // staging slot
    int it = 0;
    uint32_t store_ctr = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++it) {
      const int acc = it & 1;
      const uint32_t acc_phase = (it >> 1) & 1;
      const int m_blk = tile / args.tiles_n, n_blk = tile % args.tiles_n;
      const int m0 = m_blk * BM, n0 = n_blk * BN;
      const int row = m0 + q * 32 + lane;
      const bool row_ok = row < args.M;

      int tp = -1;
      int32_t cls = -1;
      if (KIND == KIND_FWD && row_ok) tp = __ldg(args.tpos + row);
      if (KIND == KIND_DW && row_ok) cls = __ldg(args.cand + row);

      if (!warp_wait(&tfull[acc], acc_phase, abort_flag, args.status, KIND)) break;
      tc_fence_after();

      const uint32_t t_row = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN);
      const int n_chunks = min(BN / 64, (args.N - n0 + 63) / 64);
      float m_run = -INFINITY, s_run = 0.f, z_target = 0.f;
      bool has_target = false;

      for (int c = 0; c < n_chunks; ++c) {
        const int col0 = n0 + c * 64;
        uint32_t r0[32], r1[32];
        tmem_ld32(t_row + c * 64, r0);
        tmem_ld32(t_row + c * 64 + 32, r1);
        tmem_wait_ld();
        if (c == n_chunks - 1) {
          // all TMEM reads of this accumulator are done: hand it back
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&tempty[acc]);
        }
        float v[64];
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          v[j] = __uint_as_float(r0[j]);
          v[32 + j] = __uint_as_float(r1[j]);
        }

        if (KIND == KIND_FWD) {
          const int nvalid = min(64, args.N - col0);
          float mc = -INFINITY;
          if (nvalid == 64) {
#pragma unroll
            for (int j = 0; j < 64; ++j) mc = fmaxf(mc, v[j]);
          } else {
#pragma unroll
            for (int j = 0; j < 64; ++j)
              if (j < nvalid) mc = fmaxf(mc, v[j]);
          }
          const float m_new = fmaxf(m_run, mc);
          const float mb = m_new * LOG2E;
          float sc = 0.f;
          if (nvalid == 64) {
#pragma unroll
            for (int j = 0; j < 64; ++j) sc += ex2_approx(fmaf(v[j], LOG2E, -mb));
          } else {
#pragma unroll
            for (int j = 0; j < 64; ++j)
              if (j < nvalid) sc += ex2_approx(fmaf(v[j], LOG2E, -mb));
          }
          s_run = s_run * ex2_approx((m_run - m_new) * LOG2E) + sc;
          m_run = m_new;
          const int tj = tp - col0;
          const bool mine = (tj >= 0) && (tj < nvalid);
          if (__any_sync(0xffffffffu, mine)) {
            float sel = 0.f;
#pragma unroll
            for (int j = 0; j < 64; ++j) sel = (j == tj) ? v[j] : sel;
            if (mine) {
              z_target = sel;
              has_target = true;
            }
          }
        }

        if (KIND == KIND_FWD || KIND == KIND_DX) {
          // bf16 tile -> swizzled staging box -> TMA store
          uint8_t* buf = epi_smem + (e * 2 + (store_ctr & 1)) * EPI_BUF;
          if (lane == 0) bulk_wait_read<1>();
          __syncwarp();
          const uint32_t base = smem_u32(buf) + lane * 128;
#pragma unroll
          for (int cc = 0; cc < 8; ++cc) {
            st_shared_v4(base + ((cc ^ (lane & 7)) << 4), pack_bf16x2(v[cc * 8 + 0], v[cc * 8 + 1]),
                         pack_bf16x2(v[cc * 8 + 2], v[cc * 8 + 3]),
                         pack_bf16x2(v[cc * 8 + 4], v[cc * 8 + 5]),
                         pack_bf16x2(v[cc * 8 + 6], v[cc * 8 + 7]));
          }
          fence_async_smem();
          __syncwarp();
          if (lane == 0 && m0 + q * 32 < args.M) {
            tma_store_2d(&tma_c, buf, col0, m0 + q * 32);
            bulk_commit();
          }
          ++store_ctr;
        } else {  // KIND_DW: row `row` of dW_C goes to row cand[row] of dW
          if (row_ok && cls >= 0 && cls < args.V) {
            uint4* dst = reinterpret_cast<uint4*>(args.dW + (size_t)cls * args.N + col0);
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

      if (KIND == KIND_FWD && row_ok) {
        args.stats[(size_t)n_blk * args.M + row] = make_float2(m_run, s_run);
        if (has_target) args.zt[row] = z_target;
      }
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
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

int gemm_smem_bytes() { return SMEM_BYTES; }

const void* gemm_kernel_ptr(int kind) {
  switch (kind) {
    case KIND_FWD: return reinterpret_cast<const void*>(&k_gemm<KIND_FWD>);
    case KIND_DX: return reinterpret_cast<const void*>(&k_gemm<KIND_DX>);
    default: return reinterpret_cast<const void*>(&k_gemm<KIND_DW>);
  }
}

cudaError_t launch_gemm(int kind, const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& c,
                        const GemmArgs& args, int grid, cudaStream_t s) {
  dim3 g(grid), blk(NUM_THREADS);
  switch (kind) {
    case KIND_FWD: k_gemm<KIND_FWD><<<g, blk, SMEM_BYTES, s>>>(a, b, c, args); break;
    case KIND_DX: k_gemm<KIND_DX><<<g, blk, SMEM_BYTES, s>>>(a, b, c, args); break;
    default: k_gemm<KIND_DW><<<g, blk, SMEM_BYTES, s>>>(a, b, c, args); break;
  }
  return cudaGetLastError();
}

}  // namespace ssb
