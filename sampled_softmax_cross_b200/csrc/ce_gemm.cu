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
// Work unit: a 256 x 256 output tile computed by a CTA pair (a cluster of two
// CTAs on one TPC, tcgen05 cta_group::2). Each CTA loads its own 128 rows of A
// and its 128-column half of B; the pair's leader issues M=256, N=256, K=16
// MMAs that read both CTAs' shared memory and write 128 rows x 256 fp32
// columns into each CTA's TMEM. Per CTA, 192 threads, persistent over tiles:
//   warp 0      TMA producer, 6-stage ring of 32 KB (A 128x64 + B 128x64)
//   warp 1      TMEM owner (2 x 256 columns); in the leader, the MMA issuer
//   warps 2..5  epilogue: TMEM -> registers -> math -> shared -> TMA store
//   warps 6..9  forward only: converter warps (below)
//   warp 10     forward only: publisher of finished tiles (below)
// Two TMEM accumulators let the epilogue of tile i overlap the MMAs of i+1.
//
// The forward also produces the gradient of the loss w.r.t. the logits
// ("Learning Triton ... Softmax", section "Gradient": softmax minus one-hot),
// without a separate pass. The epilogue stores, instead of the logits,
// E = exp(z - m_t) in bf16 with m_t the row's max over the 256-column tile t
// (a first pass over TMEM finds it), and the tile's (m_t, sum_j E). Once every
// tile of a 128-row half-stripe has been stored (a per-half-stripe counter,
// bumped after the TMA stores complete), converter warps merge the stripe's
// (m_t, sum) pairs into lse, write lse and the rows' losses, and rewrite E in
// place as U = E * exp(m_t - lse) - onehot (0 on ignored rows): one multiply
// per element, no exponentials. The stripe was written moments before, so
// those reads mostly hit L2. The backward GEMMs read U and scale their
// outputs by g / n.
//
// Publishing a tile stays off the epilogue's critical path: each epilogue
// warp only bumps its own shared-memory counter (release, CTA scope) once the
// TMA stores of its previous tile have completed; the publisher warp waits
// for all four counters, issues one GPU-scope fence and increments the tile
// counter of the tile's half-stripe in global memory.
#include "sm100.cuh"
#include "ss_internal.h"

namespace ssb {

constexpr int BM = 128;          // rows per CTA (256 per pair)
constexpr int BN = 256;          // output columns per tile
constexpr int BNH = BN / 2;      // B columns held by each CTA of the pair
constexpr int BK = 64, STAGES = 6;
constexpr int A_STAGE = BM * BK * 2;   // 16 KB
constexpr int B_STAGE = BNH * BK * 2;  // 16 KB
constexpr int STAGE_BYTES = A_STAGE + B_STAGE;
constexpr int EPI_BUF = 32 * 64 * 2;  // one 32-row x 64-column bf16 box (4 KB)
constexpr int EPI_BYTES = 4 * 2 * EPI_BUF;
constexpr int BAR_BYTES = 256;
constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + EPI_BYTES + BAR_BYTES;
constexpr uint32_t TMEM_COLS = 2 * BN;
constexpr float LOG2E = 1.4426950408889634f;

static_assert(SMEM_BYTES <= 232448, "shared memory budget");

template <int KIND>
struct Op;
template <>
struct Op<KIND_FWD> {  // A = x (K-major), B = W_C (K-major); 4 converter warps
  static constexpr int A_MN = 0, B_MN = 0, CONV_WARPS = 4;
};
template <>
struct Op<KIND_DX> {  // A = U (K-major), B = W_C viewed [K=P][N=d] (MN-major)
  static constexpr int A_MN = 0, B_MN = 1, CONV_WARPS = 0;
};
template <>
struct Op<KIND_DW> {  // A = U viewed [K=T][M=P] (MN-major), B = x viewed [K=T][N=d] (MN-major)
  static constexpr int A_MN = 1, B_MN = 1, CONV_WARPS = 0;
};
template <int KIND>
constexpr int num_threads() {  // + converter warps and one publisher warp
  return 192 + 32 * Op<KIND>::CONV_WARPS + (Op<KIND>::CONV_WARPS ? 32 : 0);
}

SS_DEV float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
SS_DEV float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Merge two (max, sum of exp(z - max)) pairs.
SS_DEV void merge_ms(float& m, float& s, float m2, float s2) {
  if (m2 == -INFINITY) return;
  if (m == -INFINITY) {
    m = m2;
    s = s2;
    return;
  }
  const float M = fmaxf(m, m2);
  s = s * ex2_approx((m - M) * LOG2E) + s2 * ex2_approx((m2 - M) * LOG2E);
  m = M;
}

// Converter warp: rows [r0, r0 + kRowsPerItem) of a half-stripe whose tiles
// are all stored. The stored values are E = exp(z - m_t) per 256-column tile
// t with the tile's row max m_t (from the epilogue), so
//   softmax = E * exp(m_t - lse),  lse = log sum_t exp(m_t) * s_t.
// Writes lse, the item's (loss sum, valid rows), and U = softmax - onehot.
constexpr int kConvH = 8;  // vectors per lane per half batch (two half batches in flight)

struct ConvBatch {
  uint4 in[kConvH];
  float mt;  // lane k < kConvH: m_t of the batch's k-th tile
};

SS_DEV void conv_load(const GemmArgs& args, const uint4* row, int vpr, int r, int b, ConvBatch& cb) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int k = 0; k < kConvH; ++k) {
    const int v = b * 32 * kConvH + 32 * k + lane;
    if (v < vpr) cb.in[k] = __ldcg(row + v);
  }
  const int t = b * kConvH + lane;  // 32 vectors (256 columns) per tile
  cb.mt = (lane < kConvH && t < args.tiles_n) ? __ldcg(args.stats + (size_t)t * args.M + r).x : 0.f;
}

SS_DEV void conv_store(const GemmArgs& args, uint4* row, int vpr, int b, const ConvBatch& cb, float l2,
                       int tv, int tpl) {
  const int lane = threadIdx.x & 31;
  const float f_lane = ex2_approx(fmaf(cb.mt, LOG2E, -l2));  // lane k: factor of tile k
  const int tail = args.N >> 3;  // first vector that holds a column >= N (if any)
#pragma unroll
  for (int k = 0; k < kConvH; ++k) {
    const float f = __shfl_sync(0xffffffffu, f_lane, k);
    const int v = b * 32 * kConvH + 32 * k + lane;
    if (v < vpr) {
      uint4 o;
      if (v != tv && v < tail) {
        // packed bf16x2 products: E * f rounded to bf16
        const __nv_bfloat162 f2 = __float2bfloat162_rn(f);
        const __nv_bfloat162* e2 = reinterpret_cast<const __nv_bfloat162*>(&cb.in[k]);
        __nv_bfloat162* o2 = reinterpret_cast<__nv_bfloat162*>(&o);
#pragma unroll
        for (int h = 0; h < 4; ++h) o2[h] = __hmul2(e2[h], f2);
      } else {
        // the vector holding the target column, or a ragged end: fp32 path
        const uint32_t w[4] = {cb.in[k].x, cb.in[k].y, cb.in[k].z, cb.in[k].w};
        float a[8];
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          a[2 * h] = bf16_lo(w[h]) * f;
          a[2 * h + 1] = bf16_hi(w[h]) * f;
        }
#pragma unroll
        for (int h = 0; h < 8; ++h) {
          if (v == tv && h == tpl) a[h] -= 1.f;
          if (v * 8 + h >= args.N) a[h] = 0.f;
        }
        o = make_uint4(pack_bf16x2(a[0], a[1]), pack_bf16x2(a[2], a[3]), pack_bf16x2(a[4], a[5]),
                       pack_bf16x2(a[6], a[7]));
      }
      row[v] = o;
    }
  }
}

SS_DEV void convert_item(const GemmArgs& args, int item) {
  const int lane = threadIdx.x & 31;
  const int r0 = item * kRowsPerItem;
  const int vpr = (int)(args.ldz >> 3);  // 16-byte vectors per row
  const int nb = (vpr + 32 * kConvH - 1) / (32 * kConvH);
  double lsum = 0.0;
  int lcnt = 0;
  for (int rr = 0; rr < kRowsPerItem; ++rr) {
    const int r = r0 + rr;
    if (r >= args.M) break;
    float m = -INFINITY, s = 0.f;
    for (int t = lane; t < args.tiles_n; t += 32) {
      const float2 p = __ldcg(args.stats + (size_t)t * args.M + r);
      merge_ms(m, s, p.x, p.y);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
      const float s2 = __shfl_xor_sync(0xffffffffu, s, o);
      merge_ms(m, s, m2, s2);
    }
    m = __shfl_sync(0xffffffffu, m, 0);
    s = __shfl_sync(0xffffffffu, s, 0);
    const float lse = m + logf(s);
    const int tp = __ldg(args.tpos + r);
    const bool valid = tp >= 0 && tp < args.N;
    if (lane == 0) {
      args.lse[r] = lse;
      if (valid) {
        lsum += (double)lse - (double)__ldcg(args.zt + r);
        ++lcnt;
      }
    }
    uint4* row = reinterpret_cast<uint4*>(args.u + (size_t)r * args.ldz);
    if (!valid) {
      for (int v = lane; v < vpr; v += 32) row[v] = make_uint4(0, 0, 0, 0);
      continue;
    }
    const float l2 = lse * LOG2E;
    // two half batches in flight: load b+1 while b is scaled and stored
    ConvBatch c0, c1;
    conv_load(args, row, vpr, r, 0, c0);
    for (int b = 0; b < nb; b += 2) {
      if (b + 1 < nb) conv_load(args, row, vpr, r, b + 1, c1);
      conv_store(args, row, vpr, b, c0, l2, tp >> 3, tp & 7);
      if (b + 1 < nb) {
        if (b + 2 < nb) conv_load(args, row, vpr, r, b + 2, c0);
        conv_store(args, row, vpr, b + 1, c1, l2, tp >> 3, tp & 7);
      }
    }
  }
  if (lane == 0) {
    args.partials[2 * item] = lsum;
    args.partials[2 * item + 1] = (double)lcnt;
  }
}

// Forward epilogue warp: record that its previous tile is complete (its TMA
// stores, row statistics and target logits), once at most `groups_left` of
// lane 0's bulk groups -- the current tile's -- may still be pending.
SS_DEV void epilogue_tile_done(int* warp_done, int groups_left) {
  if ((threadIdx.x & 31) == 0) {
    bulk_wait_at_most(groups_left);
    fence_async_global();
  }
  __syncwarp();
  if ((threadIdx.x & 31) == 0) red_release_cta_shared_add(warp_done, 1);
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

template <int KIND>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(num_threads<KIND>(), 1)
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
  int* epi_done = reinterpret_cast<int*>(tmem_holder + 2);  // [4] tiles completed per epilogue warp

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0 = the pair's leader
  const int cluster = blockIdx.x >> 1, num_clusters = gridDim.x >> 1;
  const int num_tiles = args.tiles_m * args.tiles_n;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);   // leader: one expect-tx arrival for both CTAs' bytes
      mbar_init(&empty[s], 1);  // one multicast commit from the leader's MMA
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);   // one multicast commit per finished accumulator
      mbar_init(&tempty[a], 8);  // leader: 4 epilogue warps of each CTA
    }
    *abort_flag = 0;
    for (int w = 0; w < 4; ++w) epi_done[w] = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_holder, TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();  // barriers of both CTAs initialised, TMEM allocated
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
    for (int tile = cluster; ok && tile < num_tiles; tile += num_clusters) {
      const int m0 = (tile / args.tiles_n) * (2 * BM) + (int)rank * BM;
      const int nh0 = (tile % args.tiles_n) * BN + (int)rank * BNH;
      for (int kb = 0; kb < args.num_kb; ++kb) {
        if (!warp_wait(&empty[stage], phase ^ 1u, abort_flag, args.status, KIND)) {
          ok = false;
          break;
        }
        if (lane == 0) {
          uint8_t* sa = smem + stage * STAGE_BYTES;
          uint8_t* sb = sa + A_STAGE;
          const int k0 = kb * BK;
          if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * STAGE_BYTES);
          const uint32_t bar = mapa_shared(smem_u32(&full[stage]), 0);
          if (Op<KIND>::A_MN) {
            tma_load_2d_pair(sa, &tma_a, bar, m0, k0);
            tma_load_2d_pair(sa + 8192, &tma_a, bar, m0 + 64, k0);
          } else {
            tma_load_2d_pair(sa, &tma_a, bar, k0, m0);
          }
          if (Op<KIND>::B_MN) {
            tma_load_2d_pair(sb, &tma_b, bar, nh0, k0);
            tma_load_2d_pair(sb + 8192, &tma_b, bar, nh0 + 64, k0);
          } else {
            tma_load_2d_pair(sb, &tma_b, bar, k0, nh0);
          }
        }
        __syncwarp();
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
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
      constexpr uint32_t IDESC = idesc_bf16(2 * BM, BN, Op<KIND>::A_MN, Op<KIND>::B_MN);
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      for (int tile = cluster; ok && tile < num_tiles; tile += num_clusters, ++it) {
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
              umma_bf16_pair(d_tmem, ad, bd, IDESC, (kb | kk) != 0 ? 1u : 0u);
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
      }
    }
  } else if (warp < 6) {
    // ----------------------------------------------------------- epilogue --
    const int q = warp & 3;   // TMEM lane quarter this warp may access
    const int e = warp - 2;   // staging slot
    int it = 0;
    uint32_t store_ctr = 0;
    float scale = 1.f;  // dX / dW: g / n (0 when no row is valid)
    if (KIND != KIND_FWD) {
      const int nv = __ldg(args.n_valid);
      scale = nv > 0 ? __ldg(args.grad_loss) / (float)nv : 0.f;
    }
    bool pending = false;  // forward: previous tile not yet recorded as complete
    for (int tile = cluster; tile < num_tiles; tile += num_clusters, ++it) {
      const int acc = it & 1;
      const uint32_t acc_phase = (it >> 1) & 1;
      const int m_blk = tile / args.tiles_n, n_blk = tile % args.tiles_n;
      const int m0 = m_blk * (2 * BM) + (int)rank * BM, n0 = n_blk * BN;
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
      int tile_groups = 0;
      float m_tile = -INFINITY, s_tile = 0.f, z_target = 0.f;
      bool has_target = false;
      if (KIND == KIND_FWD) {
        // pass 1 over TMEM: the row's max over this tile and its target logit
        for (int c = 0; c < n_chunks; ++c) {
          const int col0 = n0 + c * 64;
          uint32_t r0[32], r1[32];
          tmem_ld32(t_row + c * 64, r0);
          tmem_ld32(t_row + c * 64 + 32, r1);
          tmem_wait_ld();
          const int nvalid = min(64, args.N - col0);
          float mx[8];  // independent partial maxima (short dependency chains)
#pragma unroll
          for (int u = 0; u < 8; ++u) mx[u] = -INFINITY;
          if (nvalid == 64) {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              mx[j & 7] = fmaxf(mx[j & 7], __uint_as_float(r0[j]));
              mx[j & 7] = fmaxf(mx[j & 7], __uint_as_float(r1[j]));
            }
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              if (j < nvalid) mx[j & 7] = fmaxf(mx[j & 7], __uint_as_float(r0[j]));
              if (32 + j < nvalid) mx[j & 7] = fmaxf(mx[j & 7], __uint_as_float(r1[j]));
            }
          }
#pragma unroll
          for (int u = 0; u < 8; ++u) m_tile = fmaxf(m_tile, mx[u]);
          const int tj = tp - col0;
          const bool mine = (tj >= 0) && (tj < nvalid);
          if (__any_sync(0xffffffffu, mine)) {
            float sel = 0.f;
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              sel = (j == tj) ? __uint_as_float(r0[j]) : sel;
              sel = (32 + j == tj) ? __uint_as_float(r1[j]) : sel;
            }
            if (mine) {
              z_target = sel;
              has_target = true;
            }
          }
        }
      }
      const float mb = m_tile * LOG2E;

      for (int c = 0; c < n_chunks; ++c) {
        const int col0 = n0 + c * 64;
        uint32_t r0[32], r1[32];
        tmem_ld32(t_row + c * 64, r0);
        tmem_ld32(t_row + c * 64 + 32, r1);
        tmem_wait_ld();
        if (c == n_chunks - 1) {
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
        if (KIND != KIND_FWD) {
#pragma unroll
          for (int j = 0; j < 64; ++j) v[j] *= scale;
        }

        if (KIND == KIND_FWD) {
          // E = exp(z - m_tile) in (0, 1]: stored in place of the logits; its
          // row sum (fp32) is the tile's softmax denominator
          const int nvalid = min(64, args.N - col0);
          float sp[8];  // independent partial sums (short dependency chains)
#pragma unroll
          for (int u = 0; u < 8; ++u) sp[u] = 0.f;
          if (nvalid == 64) {
#pragma unroll
            for (int j = 0; j < 64; ++j) {
              v[j] = ex2_approx(fmaf(v[j], LOG2E, -mb));
              sp[j & 7] += v[j];
            }
          } else {
#pragma unroll
            for (int j = 0; j < 64; ++j) {
              v[j] = j < nvalid ? ex2_approx(fmaf(v[j], LOG2E, -mb)) : 0.f;
              sp[j & 7] += v[j];
            }
          }
          s_tile += ((sp[0] + sp[1]) + (sp[2] + sp[3])) + ((sp[4] + sp[5]) + (sp[6] + sp[7]));
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
            ++tile_groups;
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

      if (KIND == KIND_FWD) {
        if (row_ok) {
          args.stats[(size_t)n_blk * args.M + row] = make_float2(m_tile, s_tile);
          if (has_target) args.zt[row] = z_target;
        }
        // the previous tile's stores are done once at most this tile's are pending
        if (pending) epilogue_tile_done(epi_done + e, tile_groups);
        pending = true;
      }
    }
    if (KIND == KIND_FWD && pending) epilogue_tile_done(epi_done + e, 0);
    if (lane == 0) bulk_wait<0>();
    __syncwarp();
  } else if (warp == 10) {
    // ----------------------------------------------- publisher (forward) --
    if (KIND == KIND_FWD) {
      int k = 0;
      bool ok = true;
      for (int tile = cluster; ok && tile < num_tiles; tile += num_clusters, ++k) {
        if (lane == 0) {
          const unsigned long long t0 = globaltimer();
          for (int w = 0; w < 4 && ok; ++w) {
            while (ld_acquire_cta_shared(epi_done + w) <= k) {
              if (*abort_flag || globaltimer() - t0 > kWaitLimitNs) {
                ok = false;
                break;
              }
              __nanosleep(64);
            }
          }
          if (ok) {
            __threadfence();
            red_release_add(args.done + (tile / args.tiles_n) * 2 + (int)rank, 1);
          }
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      }
      if (!ok) raise_abort(abort_flag, args.status, KIND);
    }
  } else {
    // ------------------------------------------- converter warps (forward) --
    if (KIND == KIND_FWD) {
      while (true) {
        int item = 0;
        if (lane == 0) item = atomicAdd(args.ticket, 1);
        item = __shfl_sync(0xffffffffu, item, 0);
        if (item >= args.num_items) break;
        const int h = (item * kRowsPerItem) / BM;
        if (!wait_counter(args.done + h, args.tiles_n, abort_flag)) {
          raise_abort(abort_flag, args.status, KIND);
          break;
        }
        convert_item(args, item);
      }
    }
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

int gemm_smem_bytes() { return SMEM_BYTES; }

int gemm_rows_per_tile() { return 2 * BM; }

const void* gemm_kernel_ptr(int kind) {
  switch (kind) {
    case KIND_FWD: return reinterpret_cast<const void*>(&k_gemm<KIND_FWD>);
    case KIND_DX: return reinterpret_cast<const void*>(&k_gemm<KIND_DX>);
    default: return reinterpret_cast<const void*>(&k_gemm<KIND_DW>);
  }
}

// How many CTA pairs of this kernel can be resident at once on the device.
static int threads_of(int kind) {
  return kind == KIND_FWD ? num_threads<KIND_FWD>() : num_threads<KIND_DX>();
}

int gemm_max_pairs(int kind, int sms) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * (sms / 2));
  cfg.blockDim = dim3(threads_of(kind));
  cfg.dynamicSmemBytes = SMEM_BYTES;
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
  dim3 g(2 * pairs), blk(threads_of(kind));
  switch (kind) {
    case KIND_FWD: k_gemm<KIND_FWD><<<g, blk, SMEM_BYTES, s>>>(a, b, c, args); break;
    case KIND_DX: k_gemm<KIND_DX><<<g, blk, SMEM_BYTES, s>>>(a, b, c, args); break;
    default: k_gemm<KIND_DW><<<g, blk, SMEM_BYTES, s>>>(a, b, c, args); break;
  }
  return cudaGetLastError();
}

}  // namespace ssb
