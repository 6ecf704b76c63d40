// ce_kernels.cu -- the memory- and latency-bound steps of the sampled-softmax
// CE head: candidate build, row gather, reference logits, the row pass after
// the forward GEMM (lse, loss terms, gradient scales), the exact fix-up of
// overflowing rows, the loss reduction and the zero rows of the dense
// lm_head gradient.
#include <limits.h>

#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "sm100.cuh"
#include "ss_internal.h"

namespace ssb {

__host__ __device__ __forceinline__ int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }
__host__ __device__ __forceinline__ int64_t max64(int64_t a, int64_t b) { return a > b ? a : b; }
constexpr int kBuildThreads = 1024;

// ----------------------------------------------------------------------------
// Candidate build (sampled_softmax.py, CandidateBuilder.build / _negatives)
// ----------------------------------------------------------------------------

// Exclusive prefix sum over the block; *total receives the block sum.
__device__ int block_exclusive_scan(int x, int* total, int* s_warp) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int nwarps = (blockDim.x + 31) >> 5;
  int inc = x;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += y;
  }
  if (lane == 31) s_warp[wid] = inc;
  __syncthreads();
  if (wid == 0) {
    int w = lane < nwarps ? s_warp[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    s_warp[lane] = w;
  }
  __syncthreads();
  const int before = wid > 0 ? s_warp[wid - 1] : 0;
  *total = s_warp[nwarps - 1];
  __syncthreads();
  return before + inc - x;
}

__device__ __forceinline__ void write_status(int32_t* st, int code, int D, int need, int fallback,
                                             int draw, int next_off, int bad, int marked) {
  st[0] = code;
  st[1] = D;
  st[2] = need;
  st[3] = fallback;
  st[4] = draw;
  st[5] = next_off;
  st[6] = bad;
  st[7] = marked;
  for (int i = 8; i < SS_DEV_STATUS_WORDS; ++i) st[i] = 0;
}

__device__ __forceinline__ uint32_t ld_dsmem_u32(uint32_t cluster_addr) {
  uint32_t v;
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(cluster_addr) : "memory");
  return v;
}

// A cluster of kBuildCluster CTAs marks the targets, each its share into its
// own shared-memory bitmap; CTA 0 then ORs the others' bitmaps in (distributed
// shared memory) and alone goes on: D, negative window or fallback, and the
// bitmap with its per-word exclusive popcount prefix to global.
constexpr int kBuildCluster = 8;

__global__ void __cluster_dims__(kBuildCluster, 1, 1) __launch_bounds__(kBuildThreads)
    k_build_mark(const int32_t* __restrict__ targets, int64_t T, int32_t V, int32_t P,
                 int64_t offset, int32_t stride, uint32_t* __restrict__ g_bitmap,
                 int32_t* __restrict__ g_prefix, int32_t* __restrict__ st) {
  pdl_wait();  // the previous kernel on the stream has completed
  pdl_trigger();
  extern __shared__ uint32_t bm[];
  __shared__ int s_warp[32];
  __shared__ int s_bad;
  const int tid = threadIdx.x;
  const int NW = (V + 31) >> 5;
  const uint32_t crank = cluster_ctarank();

  for (int w = tid; w < NW; w += kBuildThreads) bm[w] = 0u;
  if (tid == 0) s_bad = INT_MAX;
  __syncthreads();

  // 1. mark this CTA's share of the valid targets (-1 = ignored; anything
  //    else outside [0, V) is an error)
  {
    const int64_t n4 = T >> 2;
    const int64_t v_lo = n4 * crank / kBuildCluster, v_hi = n4 * (crank + 1) / kBuildCluster;
    const int4* t4 = reinterpret_cast<const int4*>(targets);
    // 8 vector loads in flight per thread before the shared-memory atomics
    for (int64_t i0 = v_lo + tid; i0 < v_hi; i0 += 8 * kBuildThreads) {
      int4 q[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int64_t i = i0 + (int64_t)u * kBuildThreads;
        q[u] = i < v_hi ? __ldg(t4 + i) : make_int4(-1, -1, -1, -1);
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int64_t i = i0 + (int64_t)u * kBuildThreads;
        const int tv[4] = {q[u].x, q[u].y, q[u].z, q[u].w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int t = tv[j];
          if (t == -1) continue;
          if (t < -1 || t >= V) {
            atomicMin(&s_bad, (int)min64(4 * i + j, INT_MAX));
            continue;
          }
          const uint32_t bit = 1u << (t & 31);
          if (!(bm[t >> 5] & bit)) atomicOr(&bm[t >> 5], bit);  // frequent classes: mostly set already
        }
      }
    }
    for (int64_t i = 4 * n4 + tid; crank == 0 && i < T; i += kBuildThreads) {
      const int t = __ldg(targets + i);
      if (t == -1) continue;
      if (t < -1 || t >= V) {
        atomicMin(&s_bad, (int)min64(i, INT_MAX));
        continue;
      }
      atomicOr(&bm[t >> 5], 1u << (t & 31));
    }
  }
  __syncthreads();
  cluster_sync();  // every CTA's marks are in its shared memory
  if (crank == 0) {
    for (int w = tid; w < NW; w += kBuildThreads) {
      uint32_t v = bm[w];
      const uint32_t a = smem_u32(&bm[w]);
#pragma unroll
      for (int r = 1; r < kBuildCluster; ++r) v |= ld_dsmem_u32(mapa_shared(a, r));
      bm[w] = v;
    }
    if (tid > 0 && tid < kBuildCluster)
      atomicMin(&s_bad, (int)ld_dsmem_u32(mapa_shared(smem_u32(&s_bad), tid)));
  }
  cluster_sync();  // CTA 0 has read the others' shared memory
  if (crank != 0) return;
  if (s_bad != INT_MAX) {
    if (tid == 0) write_status(st, SS_ERR_BAD_TARGET, 0, 0, 0, 0, (int)offset, s_bad, 0);
    return;
  }

  // Each thread owns a contiguous run of bitmap words.
  const int wper = (NW + kBuildThreads - 1) / kBuildThreads;
  const int w_lo = min(NW, tid * wper), w_hi = min(NW, w_lo + wper);
  const uint32_t last_mask = (V & 31) ? ((1u << (V & 31)) - 1u) : 0xffffffffu;

  // 2. D = number of distinct valid targets
  int local = 0;
  for (int w = w_lo; w < w_hi; ++w) local += __popc(bm[w]);
  int D;
  block_exclusive_scan(local, &D, s_warp);
  if (D > P) {
    if (tid == 0) write_status(st, SS_ERR_TOO_MANY_TARGETS, D, 0, 0, 0, (int)offset, -1, D);
    return;
  }
  const int need = P - D;
  int draw = 0, fallback = 0;

  if (need > 0) {
    // 3. window of the stride sweep: positions offset .. offset+draw-1 (mod V)
    draw = (int)min64((int64_t)V, (17LL * need) / 10 + 256);
    const int kper = (draw + kBuildThreads - 1) / kBuildThreads;
    const int k_lo = min(draw, tid * kper), k_hi = min(draw, k_lo + kper);
    const int64_t smod = (int64_t)stride % V;
    int64_t k0 = offset + k_lo;
    if (k0 >= V) k0 -= V;
    const int cls0 = (int)(((int64_t)stride % V) * k0 % V);

    int cnt = 0;
    {
      int c = cls0;
      for (int k = k_lo; k < k_hi; ++k) {
        cnt += ((bm[c >> 5] >> (c & 31)) & 1u) ? 0 : 1;
        c += (int)smod;
        if (c >= V) c -= V;
      }
    }
    int total;
    const int base = block_exclusive_scan(cnt, &total, s_warp);
    if (total >= need) {
      // first `need` unmarked classes in sweep order. Classes in the window
      // are distinct, so marking one never changes another's test.
      int c = cls0, r = base;
      for (int k = k_lo; k < k_hi && r < need; ++k) {
        if (!((bm[c >> 5] >> (c & 31)) & 1u)) {
          atomicOr(&bm[c >> 5], 1u << (c & 31));
          ++r;
        }
        c += (int)smod;
        if (c >= V) c -= V;
      }
    } else {
      // fallback: evenly strided pick over the ascending unmarked classes
      fallback = 1;
      const int F = V - D;
      if (F < need) {
        if (tid == 0) write_status(st, SS_ERR_NO_FREE_CLASSES, D, need, 1, draw, (int)offset, -1, D);
        return;
      }
      const int step = max(1, F / need);
      int fcnt = 0;
      for (int w = w_lo; w < w_hi; ++w)
        fcnt += __popc(~bm[w] & (w == NW - 1 ? last_mask : 0xffffffffu));
      int ftotal;
      int r = block_exclusive_scan(fcnt, &ftotal, s_warp);
      for (int w = w_lo; w < w_hi; ++w) {
        uint32_t freeb = ~bm[w] & (w == NW - 1 ? last_mask : 0xffffffffu);
        uint32_t pick = 0u;
        while (freeb) {
          const int b = __ffs(freeb) - 1;
          freeb &= freeb - 1u;
          if (r % step == 0 && r / step < need) pick |= 1u << b;
          ++r;
        }
        bm[w] |= pick;
      }
    }
  }
  __syncthreads();

  // 4. per-word exclusive prefix of the final marks -> global
  int cnt = 0;
  for (int w = w_lo; w < w_hi; ++w) cnt += __popc(bm[w]);
  int marked;
  int run = block_exclusive_scan(cnt, &marked, s_warp);
  for (int w = w_lo; w < w_hi; ++w) {
    const uint32_t b = bm[w];
    g_bitmap[w] = b;
    g_prefix[w] = run;
    run += __popc(b);
  }
  if (tid == 0) {
    const int next_off = (int)((offset + draw) % V);
    write_status(st, marked == P ? SS_OK : SS_ERR_NO_FREE_CLASSES, D, need, fallback, draw,
                 next_off, -1, marked);
  }
}

// candidates / vocab_pos from the bitmap (threads [0, V)), target_pos (threads [V, V+T)).
__global__ void k_build_emit(const int32_t* __restrict__ targets, int64_t T, int32_t V, int32_t P,
                             const uint32_t* __restrict__ bitmap, const int32_t* __restrict__ prefix,
                             int32_t* __restrict__ st, int32_t* __restrict__ candidates,
                             int32_t* __restrict__ target_pos, int32_t* __restrict__ vocab_pos) {
  pdl_wait();  // the previous kernel on the stream has completed
  pdl_trigger();
  const int code = *reinterpret_cast<const volatile int32_t*>(st);
  const int64_t n = (int64_t)V + T;
  for (int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; g < n;
       g += (int64_t)gridDim.x * blockDim.x) {
    if (g < V) {
      const int c = (int)g;
      if (code != SS_OK) {
        vocab_pos[c] = -1;
        if (c < P) candidates[c] = -1;
        continue;
      }
      const uint32_t bits = bitmap[c >> 5];
      const int b = c & 31;
      if ((bits >> b) & 1u) {
        const int pos = prefix[c >> 5] + __popc(bits & ((1u << b) - 1u));
        vocab_pos[c] = pos;
        if (SS_CHECK(pos >= 0 && pos < P, st + 8, 1)) candidates[pos] = c;
      } else {
        vocab_pos[c] = -1;
      }
    } else {
      const int64_t i = g - V;
      const int t = __ldg(targets + i);
      if (code != SS_OK || t < 0 || t >= V) {
        target_pos[i] = -1;
        continue;
      }
      const uint32_t bits = bitmap[t >> 5];
      const int b = t & 31;
      const int pos = prefix[t >> 5] + __popc(bits & ((1u << b) - 1u));
      target_pos[i] = SS_CHECK(((bits >> b) & 1u) && pos < P, st + 8, 2) ? pos : -1;
    }
  }
}

// ----------------------------------------------------------------------------
// Row gather W_C[j] = lm_head[C_j] (sampled_softmax.py, _gather_rows): one warp
// per row, 16-byte vectors.
// ----------------------------------------------------------------------------
// Block 0 also clears `zero_words` (the forward's tile counters) for the
// kernel that follows on the stream.
__global__ void k_gather(const uint4* __restrict__ lm, const int32_t* __restrict__ cand, int32_t P,
                         int32_t vec_per_row, int32_t V, uint4* __restrict__ w_c,
                         int32_t* __restrict__ status, int32_t* __restrict__ zero_words,
                         int32_t n_zero_words) {
  pdl_wait();  // the previous kernel on the stream has completed
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  if (blockIdx.x == 0)
    for (int i = threadIdx.x; i < n_zero_words; i += blockDim.x) zero_words[i] = 0;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t r = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < P; r += warps) {
    const int c = __ldg(cand + r);
    uint4* dst = w_c + r * vec_per_row;
    if (c < 0 || c >= V) {
      for (int v = lane; v < vec_per_row; v += 32) dst[v] = make_uint4(0, 0, 0, 0);
      if (lane == 0 && atomicCAS(status, 0, (int32_t)SS_ERR_BAD_INDEX) == 0) status[1] = 1;
      continue;
    }
    const uint4* src = lm + (int64_t)c * vec_per_row;
    int v = lane;
    for (; v + 64 < vec_per_row; v += 96) {
      const uint4 a = __ldg(src + v), b = __ldg(src + v + 32), d = __ldg(src + v + 64);
      dst[v] = a;
      dst[v + 32] = b;
      dst[v + 64] = d;
    }
    for (; v < vec_per_row; v += 32) dst[v] = __ldg(src + v);
  }
}

// ----------------------------------------------------------------------------
// Reference logit per row: ref_i = x_i . W_C[target_pos_i] in fp32 (W_C[0] on
// ignored rows). The forward GEMM's epilogue stores exp(z - ref) (ce_gemm.cu).
// One warp per row; fixed summation order.
// ----------------------------------------------------------------------------
__device__ __forceinline__ float dot8_bf16(uint4 a, uint4 b, float acc) {
  const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
  for (int h = 0; h < 4; ++h) {
    acc = fmaf(__uint_as_float(wa[h] << 16), __uint_as_float(wb[h] << 16), acc);
    acc = fmaf(__uint_as_float(wa[h] & 0xffff0000u), __uint_as_float(wb[h] & 0xffff0000u), acc);
  }
  return acc;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_down_sync(0xffffffffu, v, o);
  return __shfl_sync(0xffffffffu, v, 0);
}

__global__ void k_ref_logits(const uint4* __restrict__ x, const uint4* __restrict__ w_c,
                             const int32_t* __restrict__ tpos, int64_t T, int32_t vpr, int32_t P,
                             float* __restrict__ ref) {
  pdl_wait();  // the previous kernel on the stream has completed
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int64_t pairs = (T + 1) / 2;  // two rows per warp iteration, all loads in flight
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t pi = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); pi < pairs; pi += warps) {
    float acc[2] = {0.f, 0.f};
    for (int v0 = 0; v0 < vpr; v0 += 96) {
      uint4 xa[2][3], wa[2][3];
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int64_t r = 2 * pi + k;
        const int t = r < T ? __ldg(tpos + r) : -1;
        const int j = (t >= 0 && t < P) ? t : 0;
#pragma unroll
        for (int h = 0; h < 3; ++h) {
          const int v = v0 + lane + 32 * h;
          const bool ok = r < T && v < vpr;
          xa[k][h] = ok ? __ldg(x + r * vpr + v) : make_uint4(0, 0, 0, 0);
          wa[k][h] = ok ? __ldg(w_c + (int64_t)j * vpr + v) : make_uint4(0, 0, 0, 0);
        }
      }
#pragma unroll
      for (int k = 0; k < 2; ++k)
#pragma unroll
        for (int h = 0; h < 3; ++h) acc[k] = dot8_bf16(xa[k][h], wa[k][h], acc[k]);
    }
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const float sum = warp_sum(acc[k]);
      if (lane == 0 && 2 * pi + k < T) ref[2 * pi + k] = sum;
    }
  }
}

// ----------------------------------------------------------------------------
// e4m3 (OCP 8-bit floating point, E4M3) helpers. Codes are produced by the
// hardware conversion (round to nearest even, saturating at +-448) and read
// back through fp16, which holds every e4m3 value exactly.
// ----------------------------------------------------------------------------
__device__ __forceinline__ float2 e4m3x2_to_float2(uint16_t two_codes) {
  const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(two_codes, __NV_E4M3);
  return __half22float2(*reinterpret_cast<const __half2*>(&h));
}

__device__ __forceinline__ uint16_t float2_to_e4m3x2(float lo, float hi) {
  return __nv_cvt_float2_to_fp8x2(make_float2(lo, hi), __NV_SATFINITE, __NV_E4M3);
}

// Exponent k of the per-tensor scale: the smallest k with amax <= 448 * 2^k,
// kept in [-126, 127] (2^k and 2^-k normal); 0 for an all-zero tensor.
__device__ __forceinline__ int e4m3_scale_exp(float amax) {
  if (!(amax > 0.f)) return 0;
  int ex;
  frexpf(amax, &ex);
  int k = ex - 9;
  for (int i = 0; i < 4 && amax > ldexpf(448.f, k); ++i) ++k;
  for (int i = 0; i < 4 && amax <= ldexpf(448.f, k - 1); ++i) --k;
  return min(max(k, -126), 127);
}

// amax[0] = max |a|, amax[1] = max |b| as bf16 bit patterns (monotonic in
// the magnitude for finite values), by atomicMax.
__global__ void k_amax_bf16(const uint4* __restrict__ a, int64_t na, const uint4* __restrict__ b,
                            int64_t nb, uint32_t* __restrict__ amax) {
  pdl_wait();  // the previous kernel on the stream has completed
  pdl_trigger();
  uint32_t ma = 0, mb = 0;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  constexpr int U = 4;  // independent loads in flight per thread
  for (int64_t i0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i0 < na + nb;
       i0 += U * stride) {
    uint4 v[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t i = i0 + u * stride;
      v[u] = i < na ? __ldg(a + i) : (i < na + nb ? __ldg(b + (i - na)) : make_uint4(0, 0, 0, 0));
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
      uint32_t m = 0;
#pragma unroll
      for (int h = 0; h < 4; ++h) m = max(m, max(w[h] & 0x7fffu, (w[h] >> 16) & 0x7fffu));
      if (i0 + u * stride < na)
        ma = max(ma, m);
      else
        mb = max(mb, m);
    }
  }
  // one atomic per block and tensor: per-warp atomics on one address serialise
  __shared__ uint32_t s_m[2][32];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    ma = max(ma, __shfl_xor_sync(0xffffffffu, ma, o));
    mb = max(mb, __shfl_xor_sync(0xffffffffu, mb, o));
  }
  if ((threadIdx.x & 31) == 0) {
    s_m[0][threadIdx.x >> 5] = ma;
    s_m[1][threadIdx.x >> 5] = mb;
  }
  __syncthreads();
  if (threadIdx.x < 2) {
    uint32_t m = 0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) m = max(m, s_m[threadIdx.x][w]);
    if (m) atomicMax(amax + threadIdx.x, m);
  }
}

__global__ void k_quant_e4m3(const uint4* __restrict__ a, int64_t na, uint2* __restrict__ a8,
                             const uint4* __restrict__ b, int64_t nb, uint2* __restrict__ b8,
                             const uint32_t* __restrict__ amax, float* __restrict__ qscale) {
  pdl_wait();  // the previous kernel on the stream has completed
  pdl_trigger();
  const int ka = e4m3_scale_exp(__uint_as_float(amax[0] << 16));
  const int kb = e4m3_scale_exp(__uint_as_float(amax[1] << 16));
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    qscale[0] = ldexpf(1.f, ka);
    qscale[1] = ldexpf(1.f, kb);
    qscale[2] = ldexpf(1.f, ka + kb);
  }
  const float ia = ldexpf(1.f, -ka), ib = ldexpf(1.f, -kb);  // exact: powers of two
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  constexpr int U = 4;  // independent loads in flight per thread
  for (int64_t i0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i0 < na + nb;
       i0 += U * stride) {
    uint4 v[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t i = i0 + u * stride;
      v[u] = i < na ? __ldg(a + i) : (i < na + nb ? __ldg(b + (i - na)) : make_uint4(0, 0, 0, 0));
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t i = i0 + u * stride;
      if (i >= na + nb) break;
      const bool in_a = i < na;
      const float sc = in_a ? ia : ib;
      const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
      uint16_t q[4];
#pragma unroll
      for (int h = 0; h < 4; ++h)
        q[h] = float2_to_e4m3x2(__uint_as_float(w[h] << 16) * sc,
                                __uint_as_float(w[h] & 0xffff0000u) * sc);
      const uint2 out = make_uint2((uint32_t)q[0] | ((uint32_t)q[1] << 16),
                                   (uint32_t)q[2] | ((uint32_t)q[3] << 16));
      if (in_a)
        a8[i] = out;
      else
        b8[i - na] = out;
    }
  }
}

// Reference logit for the e4m3 forward: the same dot product the GEMM forms
// (codes times the product of the two scales), fp32. One warp per row.
__global__ void k_ref_logits_e4m3(const uint4* __restrict__ x8, const uint4* __restrict__ w8,
                                  const int32_t* __restrict__ tpos, int64_t T, int32_t vpr,
                                  int32_t P, const float* __restrict__ qscale,
                                  float* __restrict__ ref) {
  pdl_wait();  // the previous kernel on the stream has completed
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  const float s = __ldg(qscale + 2);
  for (int64_t r = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < T; r += warps) {
    const int t = __ldg(tpos + r);
    const int j = (t >= 0 && t < P) ? t : 0;
    float acc = 0.f;
    for (int v = lane; v < vpr; v += 32) {
      const uint4 xa = __ldg(x8 + r * vpr + v), wa = __ldg(w8 + (int64_t)j * vpr + v);
      const uint32_t xw[4] = {xa.x, xa.y, xa.z, xa.w}, ww[4] = {wa.x, wa.y, wa.z, wa.w};
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        const float2 x0 = e4m3x2_to_float2((uint16_t)(xw[h] & 0xffffu));
        const float2 x1 = e4m3x2_to_float2((uint16_t)(xw[h] >> 16));
        const float2 w0 = e4m3x2_to_float2((uint16_t)(ww[h] & 0xffffu));
        const float2 w1 = e4m3x2_to_float2((uint16_t)(ww[h] >> 16));
        acc = fmaf(x0.x, w0.x, acc);
        acc = fmaf(x0.y, w0.y, acc);
        acc = fmaf(x1.x, w1.x, acc);
        acc = fmaf(x1.y, w1.y, acc);
      }
    }
    const float sum = warp_sum(acc);
    if (lane == 0) ref[r] = sum * s;
  }
}

// ----------------------------------------------------------------------------
// Row pass after the forward GEMM. With S_i = sum of the row's partial sums of
// exp(z - ref_i) (one per tile, or per half tile in the e4m3 forward):
//   lse_i = ref_i + log S_i,   loss_i = lse_i - z_target = log S_i (valid rows),
//   r_i = 1 / S_i (0 on ignored rows),  E'[i, t_i] = 1 - S_i,  x'_i = r_i x_i,
// so that r_i E'_ij = softmax_ij - [j == t_i] (the CE gradient w.r.t. the
// logits, "Learning Triton One Kernel at a Time: Softmax", section "Gradient")
// and the backward is dX = (g/n) r (.) (E' W_C), dW_C = (g/n) E'^T x'.
// A row whose S_i is not below 2^64 (E overflowed: its loss exceeds ~44 nats)
// is listed for the exact fix-up in k_finalize instead.
// ----------------------------------------------------------------------------
constexpr float kFixThreshold = 1.8446744e19f;  // 2^64

__device__ __forceinline__ uint4 scale_bf16x8(uint4 a, float r) {
  const uint32_t w[4] = {a.x, a.y, a.z, a.w};
  uint32_t o[4];
#pragma unroll
  for (int h = 0; h < 4; ++h)
    o[h] = pack_bf16x2(__uint_as_float(w[h] << 16) * r, __uint_as_float(w[h] & 0xffff0000u) * r);
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// Each warp takes 8 consecutive rows. For the partial sums (stored sum-major)
// lane l adds sums (l / 8), (l / 8) + 4, ... of row (l % 8), so every load
// instruction reads whole 32-byte sectors; the four lane totals of a row are
// then combined in a fixed order. The x' rows are written 4 at a time with
// all their loads in flight.
constexpr int kRowsPerWarp = 8;

__global__ void __launch_bounds__(256, 3) k_rows(RowArgs a) {
  pdl_wait();  // the previous kernel on the stream has completed
  pdl_trigger();
  __shared__ double2 s_part[8];
  const int lane = threadIdx.x & 31;
  const int vpr = a.d / 8;
  const int64_t groups = (a.T + kRowsPerWarp - 1) / kRowsPerWarp;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  double w_sum = 0.0;  // this warp's valid, non-overflowed row losses (lane 0)
  int w_cnt = 0;       // this warp's valid rows
  for (int64_t gidx = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); gidx < groups;
       gidx += warps) {
    const int64_t r = gidx * kRowsPerWarp + (lane & 7);
    const bool in = r < a.T;
    float s = 0.f;
    if (in) {
      // eight loads in flight per batch, added in the order of t
      int t = lane >> 3;
      for (; t + 28 < a.nsums; t += 32) {
        float v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) v[u] = __ldg(a.rowsum + (int64_t)(t + 4 * u) * a.T + r);
#pragma unroll
        for (int u = 0; u < 8; ++u) s += v[u];
      }
      for (; t < a.nsums; t += 4) s += __ldg(a.rowsum + (int64_t)t * a.T + r);
    }
    s += __shfl_xor_sync(0xffffffffu, s, 8);
    s += __shfl_xor_sync(0xffffffffu, s, 16);
    const float S = s;  // identical in the four lanes of the row
    const int tp = in ? __ldg(a.tpos + r) : -1;
    const bool valid = tp >= 0 && tp < a.P;
    const bool fix = in && !(S < kFixThreshold);  // overflow (or NaN): exact recomputation later
    const float rs = (in && valid && !fix) ? 1.f / S : 0.f;
    if (lane < 8) {
      if (in && fix) {
        const int k = atomicAdd(a.fix_count, 1);
        if (SS_CHECK(k < a.T, a.status, 3)) a.fix_list[k] = (int32_t)r;
      }
      if (in && !fix) {
        a.lse[r] = __ldg(a.ref + r) + logf(S);
        a.loss_rows[r] = valid ? logf(S) : 0.f;
        a.rscale[r] = rs;
        if (valid && SS_CHECK(tp < a.ldz, a.status, 4))
          a.u[r * a.ldz + tp] = (uint16_t)(pack_bf16x2(1.f - S, 0.f) & 0xffffu);
      }
    }
    {  // loss sum and valid count of the warp's 8 rows, fixed order
      double l = (lane < 8 && in && valid && !fix) ? (double)logf(S) : 0.0;
      int c = (lane < 8 && in && valid) ? 1 : 0;
#pragma unroll
      for (int o = 1; o < 8; o <<= 1) {
        l += __shfl_xor_sync(0xffffffffu, l, o);
        c += __shfl_xor_sync(0xffffffffu, c, o);
      }
      w_sum += l;
      w_cnt += c;
    }
    const unsigned todo = __ballot_sync(0xffffffffu, lane < 8 && in && !fix);
    for (int k0 = 0; k0 < kRowsPerWarp; k0 += 4) {
      uint4 in_v[4][3];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int64_t rr = gidx * kRowsPerWarp + k0 + k;
        const uint4* xr = reinterpret_cast<const uint4*>(a.x) + rr * vpr;
#pragma unroll
        for (int h = 0; h < 3; ++h) {
          const int v = lane + 32 * h;
          if (((todo >> (k0 + k)) & 1u) && v < vpr) in_v[k][h] = __ldg(xr + v);
        }
      }
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        if (!((todo >> (k0 + k)) & 1u)) continue;
        const float rk = __shfl_sync(0xffffffffu, rs, k0 + k);
        const int64_t rr = gidx * kRowsPerWarp + k0 + k;
        const uint4* xr = reinterpret_cast<const uint4*>(a.x) + rr * vpr;
        uint4* xo = reinterpret_cast<uint4*>(a.xs) + rr * vpr;
#pragma unroll
        for (int h = 0; h < 3; ++h) {
          const int v = lane + 32 * h;
          if (v < vpr) xo[v] = scale_bf16x8(in_v[k][h], rk);
        }
        for (int v = lane + 96; v < vpr; v += 32) xo[v] = scale_bf16x8(__ldg(xr + v), rk);
      }
    }
  }
  if (lane == 0) s_part[threadIdx.x >> 5] = make_double2(w_sum, (double)w_cnt);
  __syncthreads();
  if (threadIdx.x == 0) {
    double2 t = s_part[0];
    for (int w = 1; w < (int)(blockDim.x >> 5); ++w) {
      t.x += s_part[w].x;
      t.y += s_part[w].y;
    }
    a.partials[blockIdx.x] = t;
  }
}

// After the row pass, one CTA:
//  1. exact recomputation of listed rows, max-shifted (section "Definition"):
//     the row's P logits in fp32, then lse, the row loss, r_i, x'_i and the
//     row of E' with the row max as the shift;
//  2. the loss: sum of the valid rows' losses over the valid-row count
//     (Handout #16 CPU checks, lm_gradient), in a fixed order (deterministic).
//     Without listed rows it adds the row pass's per-block partial sums; with
//     them it adds every row's loss again.
constexpr int kFinThreads = 1024;

__device__ float block_reduce(float v, bool is_max, float* sh) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float w = __shfl_down_sync(0xffffffffu, v, o);
    v = is_max ? fmaxf(v, w) : v + w;
  }
  if (lane == 0) sh[wid] = v;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = sh[0];
    for (int w = 1; w < (int)(blockDim.x >> 5); ++w) t = is_max ? fmaxf(t, sh[w]) : t + sh[w];
    sh[32] = t;
  }
  __syncthreads();
  const float out = sh[32];
  __syncthreads();
  return out;
}

__device__ __forceinline__ float row_logit(const uint4* xr, const uint4* wr, int vpr) {
  float acc = 0.f;
  for (int v = 0; v < vpr; ++v) acc = dot8_bf16(__ldg(xr + v), __ldg(wr + v), acc);
  return acc;
}

// Logit of row r and class j in the row pass's precision: bf16 x . W_C, or
// for the e4m3 forward, the scales times the dot product of the codes.
__device__ __forceinline__ float row_logit_any(const RowArgs& a, int64_t r, int64_t j, int vpr) {
  if (a.x8 == nullptr)
    return row_logit(reinterpret_cast<const uint4*>(a.x) + r * vpr,
                     reinterpret_cast<const uint4*>(a.w_c) + j * vpr, vpr);
  float acc = 0.f;
  for (int k = 0; k < a.d; k += 2) {
    const float2 xf = e4m3x2_to_float2(*reinterpret_cast<const uint16_t*>(a.x8 + r * a.d + k));
    const float2 wf = e4m3x2_to_float2(*reinterpret_cast<const uint16_t*>(a.w8 + j * a.d + k));
    acc = fmaf(xf.x, wf.x, acc);
    acc = fmaf(xf.y, wf.y, acc);
  }
  return acc * __ldg(a.qscale + 2);
}

__global__ void __launch_bounds__(kFinThreads) k_finalize(RowArgs a, int32_t nparts) {
  pdl_wait();  // the previous kernel on the stream has completed
  pdl_trigger();
  __shared__ float sh[33];
  __shared__ float s_zt;
  __shared__ double s_sum[32], s_cnt[32];
  int n = *reinterpret_cast<volatile int32_t*>(a.fix_count);
  if (!SS_CHECK(n <= a.T, a.status, 5)) n = 0;
  const int vpr = a.d / 8;
  const int nt = blockDim.x;
  for (int k = 0; k < n; ++k) {
    const int64_t r = a.fix_list[k];
    if (!SS_CHECK(r >= 0 && r < a.T, a.status, 6)) continue;
    const int tp = a.tpos[r];
    const bool valid = tp >= 0 && tp < a.P;
    const uint4* xr = reinterpret_cast<const uint4*>(a.x) + r * vpr;
    float m = -INFINITY;
    for (int j = threadIdx.x; j < a.P; j += nt) m = fmaxf(m, row_logit_any(a, r, j, vpr));
    m = block_reduce(m, true, sh);
    float sum = 0.f;
    uint16_t* ur = a.u + r * a.ldz;
    for (int j = threadIdx.x; j < a.P; j += nt) {
      const float z = row_logit_any(a, r, j, vpr);
      const float e = expf(z - m);
      sum += e;
      ur[j] = valid ? (uint16_t)(pack_bf16x2(e, 0.f) & 0xffffu) : (uint16_t)0;
      if (j == tp) s_zt = z;
    }
    const float S = block_reduce(sum, false, sh);  // also orders the E' writes above
    const float rs = valid ? 1.f / S : 0.f;
    if (threadIdx.x == 0) {
      const float lse = m + logf(S);
      a.lse[r] = lse;
      a.loss_rows[r] = valid ? lse - s_zt : 0.f;
      a.rscale[r] = rs;
      if (valid) ur[tp] = (uint16_t)(pack_bf16x2(expf(s_zt - m) - S, 0.f) & 0xffffu);
    }
    uint4* xo = reinterpret_cast<uint4*>(a.xs) + r * vpr;
    for (int v = threadIdx.x; v < vpr; v += nt) xo[v] = scale_bf16x8(__ldg(xr + v), rs);
    __syncthreads();
  }

  double s = 0.0, c = 0.0;
  if (n == 0) {
    for (int i = threadIdx.x; i < nparts; i += nt) {
      const double2 p = a.partials[i];
      s += p.x;
      c += p.y;
    }
  } else {
    // each thread takes runs of 4 consecutive rows (T rounded down to a
    // multiple of 4 here; the rest below), fixed order
    const int64_t T = a.T;
    const int64_t T4 = T & ~int64_t(3);
    for (int64_t i = 4 * (int64_t)threadIdx.x; i < T4; i += 4 * (int64_t)nt) {
      const float4 l = *reinterpret_cast<const float4*>(a.loss_rows + i);
      const int4 t = __ldg(reinterpret_cast<const int4*>(a.tpos + i));
      const float lv[4] = {l.x, l.y, l.z, l.w};
      const int tv[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (tv[u] >= 0 && tv[u] < a.P) {
          s += (double)lv[u];
          c += 1.0;
        }
      }
    }
    for (int64_t i = T4 + threadIdx.x; i < T; i += nt) {
      const int t = a.tpos[i];
      if (t >= 0 && t < a.P) {
        s += (double)a.loss_rows[i];
        c += 1.0;
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    s += __shfl_down_sync(0xffffffffu, s, o);
    c += __shfl_down_sync(0xffffffffu, c, o);
  }
  if ((threadIdx.x & 31) == 0) {
    s_sum[threadIdx.x >> 5] = s;
    s_cnt[threadIdx.x >> 5] = c;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double ts = 0.0, tc = 0.0;
    for (int w = 0; w < (nt >> 5); ++w) {
      ts += s_sum[w];
      tc += s_cnt[w];
    }
    *a.n_valid = (int32_t)tc;
    *a.loss = tc > 0.0 ? (float)(ts / tc) : 0.f;
  }
}

// dW rows outside C (or every row) set to +0.0.
__global__ void k_zero_rows(uint4* __restrict__ dW, int32_t V, int32_t vec_per_row,
                            const int32_t* __restrict__ vocab_pos, int all_rows) {
  pdl_wait();  // the previous kernel on the stream has completed
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t r = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < V; r += warps) {
    if (!all_rows && __ldg(vocab_pos + r) >= 0) continue;
    uint4* dst = dW + r * vec_per_row;
    for (int v = lane; v < vec_per_row; v += 32) __stcs(dst + v, make_uint4(0, 0, 0, 0));
  }
}

// ----------------------------------------------------------------------------
// Prefix-target positions (sampled_softmax.py, CandidateBuilder.build: the
// prefix target of each token, then its position in C through the same
// class -> position map as the targets). One thread per token; a prefix class
// outside C, "no prefix" (-1) and an ignored token all give -1, so a prefix
// target never adds a class to C.
// ----------------------------------------------------------------------------
__global__ void k_prefix_pos(const int32_t* __restrict__ prefix_table,
                             const int32_t* __restrict__ targets,
                             const int32_t* __restrict__ vocab_pos, int64_t T, int32_t V,
                             int32_t* __restrict__ prefix_pos, int32_t* __restrict__ status) {
  pdl_wait();  // the previous kernel on the stream has completed
  pdl_trigger();
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < T; i += stride) {
    const int t = __ldg(targets + i);
    int pos = -1, bad = 0;
    if (t >= 0 && t < V) {
      const int p = __ldg(prefix_table + t);
      if (p >= 0 && p < V)
        pos = __ldg(vocab_pos + p);
      else if (p != -1)
        bad = 2;
    } else if (t != -1) {
      bad = 3;
    }
    if (bad && atomicCAS(status, 0, (int32_t)SS_ERR_BAD_INDEX) == 0) status[1] = bad;
    prefix_pos[i] = pos;
  }
}

// ----------------------------------------------------------------------------
// launchers
// ----------------------------------------------------------------------------
// Per-device launch facts (a process may drive several GPUs).
constexpr int kMaxDevices = 128;
static int g_sms_cache[kMaxDevices] = {};
static bool g_build_attr[kMaxDevices] = {};

static int current_device() {
  int dev = 0;
  cudaGetDevice(&dev);
  return (dev >= 0 && dev < kMaxDevices) ? dev : 0;
}

static int num_sms() {
  const int dev = current_device();
  if (g_sms_cache[dev] == 0) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    g_sms_cache[dev] = n > 0 ? n : 148;
  }
  return g_sms_cache[dev];
}

cudaError_t launch_build_mark(const int32_t* targets, int64_t T, int32_t V, int32_t P,
                              int64_t offset, int32_t stride, uint32_t* bitmap, int32_t* prefix,
                              int32_t* dev_status, cudaStream_t s) {
  const int smem = ((V + 31) / 32) * 4;
  const int dev = current_device();
  if (!g_build_attr[dev]) {  // the attribute is per device
    cudaError_t e = cudaFuncSetAttribute(k_build_mark, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (SS_MAX_VOCAB / 32) * 4);
    if (e != cudaSuccess) return e;
    g_build_attr[dev] = true;
  }
  return launch_pdl(k_build_mark, dim3(kBuildCluster), dim3(kBuildThreads), smem, s, targets, T, V, P, offset, stride,
                                                          bitmap, prefix, dev_status);
}

cudaError_t launch_build_emit(const int32_t* targets, int64_t T, int32_t V, int32_t P,
                              const uint32_t* bitmap, const int32_t* prefix,
                              int32_t* dev_status, int32_t* candidates,
                              int32_t* target_pos, int32_t* vocab_pos, cudaStream_t s) {
  const int64_t n = (int64_t)V + T;
  const int blocks = (int)min64((n + 255) / 256, (int64_t)num_sms() * 8);
  return launch_pdl(k_build_emit, dim3(blocks), dim3(256), 0, s, targets, T, V, P, bitmap, prefix, dev_status, candidates,
                                      target_pos, vocab_pos);
}

cudaError_t launch_gather(const uint16_t* lm_head, const int32_t* cand, int32_t P, int32_t d,
                          int32_t V, uint16_t* w_c, int32_t* status, int32_t* zero_words,
                          int32_t n_zero_words, cudaStream_t s) {
  const int warps_per_block = 8;
  const int blocks = (int)min64((P + warps_per_block - 1) / warps_per_block,
                                       (int64_t)num_sms() * 16);
  return launch_pdl(k_gather, dim3(blocks), dim3(warps_per_block * 32), 0, s, reinterpret_cast<const uint4*>(lm_head), cand, P,
                                                    d / 8, V, reinterpret_cast<uint4*>(w_c), status,
                                                    zero_words, n_zero_words);
}

cudaError_t launch_ref_logits(const uint16_t* x, const uint16_t* w_c, const int32_t* tpos,
                              int64_t T, int32_t d, int32_t P, float* ref, cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  const int blocks = (int)min64(((T + 1) / 2 + 7) / 8, (int64_t)num_sms() * 16);
  return launch_pdl(k_ref_logits, dim3(blocks), dim3(256), 0, s, reinterpret_cast<const uint4*>(x),
                                      reinterpret_cast<const uint4*>(w_c), tpos, T, d / 8, P, ref);
}

static int rows_blocks(int64_t T) {
  if (T == 0) return 0;
  const int64_t groups = (T + kRowsPerWarp - 1) / kRowsPerWarp;  // per warp; 8 warps per block
  return (int)min64(min64((groups + 7) / 8, (int64_t)num_sms() * 16), (int64_t)kRowPartials);
}

cudaError_t launch_rows(const RowArgs& a, cudaStream_t s) {
  const int blocks = rows_blocks(a.T);
  if (blocks == 0) return cudaSuccess;
  return launch_pdl(k_rows, dim3(blocks), dim3(256), 0, s, a);
}

cudaError_t launch_finalize(const RowArgs& a, cudaStream_t s) {
  return launch_pdl(k_finalize, dim3(1), dim3(kFinThreads), 0, s, a, rows_blocks(a.T));
}

cudaError_t launch_prefix_pos(const int32_t* prefix_table, const int32_t* targets,
                              const int32_t* vocab_pos, int64_t T, int32_t V, int32_t* prefix_pos,
                              int32_t* status, cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  const int blocks = (int)min64((T + 255) / 256, (int64_t)num_sms() * 8);
  return launch_pdl(k_prefix_pos, dim3(blocks), dim3(256), 0, s, prefix_table, targets, vocab_pos, T, V, prefix_pos, status);
}

cudaError_t launch_amax_bf16(const uint16_t* a, int64_t n, const uint16_t* b, int64_t m,
                             uint32_t* amax, cudaStream_t s) {
  const int64_t vec = (n + m) / 8;
  if (vec == 0) return cudaSuccess;
  const int blocks = (int)min64((vec + 255) / 256, (int64_t)num_sms() * 8);
  return launch_pdl(k_amax_bf16, dim3(blocks), dim3(256), 0, s, reinterpret_cast<const uint4*>(a), n / 8,
                                     reinterpret_cast<const uint4*>(b), m / 8, amax);
}

cudaError_t launch_quant_e4m3(const uint16_t* a, int64_t n, uint8_t* a8, const uint16_t* b,
                              int64_t m, uint8_t* b8, const uint32_t* amax, float* qscale,
                              cudaStream_t s) {
  const int64_t vec = (n + m) / 8;
  const int blocks = (int)max64(1, min64((vec + 255) / 256, (int64_t)num_sms() * 8));
  return launch_pdl(k_quant_e4m3, dim3(blocks), dim3(256), 0, s, reinterpret_cast<const uint4*>(a), n / 8,
                                      reinterpret_cast<uint2*>(a8),
                                      reinterpret_cast<const uint4*>(b), m / 8,
                                      reinterpret_cast<uint2*>(b8), amax, qscale);
}

cudaError_t launch_ref_logits_e4m3(const uint8_t* x8, const uint8_t* w8, const int32_t* tpos,
                                   int64_t T, int32_t d, int32_t P, const float* qscale,
                                   float* ref, cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  const int blocks = (int)min64((T + 7) / 8, (int64_t)num_sms() * 16);
  return launch_pdl(k_ref_logits_e4m3, dim3(blocks), dim3(256), 0, s, reinterpret_cast<const uint4*>(x8),
                                           reinterpret_cast<const uint4*>(w8), tpos, T, d / 16, P,
                                           qscale, ref);
}

cudaError_t launch_zero_rows(uint16_t* dW, int32_t V, int32_t d, const int32_t* vocab_pos,
                             int all_rows, cudaStream_t s) {
  const int blocks = (int)min64((V + 7) / 8, (int64_t)num_sms() * 16);
  return launch_pdl(k_zero_rows, dim3(blocks), dim3(256), 0, s, reinterpret_cast<uint4*>(dW), V, d / 8, vocab_pos, all_rows);
}

}  // namespace ssb
