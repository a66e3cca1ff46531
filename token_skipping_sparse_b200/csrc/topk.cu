// topk.cu -- token selection of SPTS (the informative tokens of Fig. 2(a)/(b)).
//
// One CTA of 1024 threads:
//   1. (MAXNORM_ADD) block maxima of both score vectors over all Nc;
//   2. fused score f per candidate in fp32, one rounding per operation
//      (w_a*(s/max s) + w_b*(c/max c), or s*c, or s), mapped to an
//      order-preserving uint32 key (-0 -> +0);
//   3. MSB-first radix select, 4 digits of 8 bits, over the first Nc - tail
//      candidates: finds the key T of the (k - tail)-th largest and how many
//      keys equal to T must be taken;
//   4. stable compaction in index order: a candidate is kept if its key > T,
//      or == T and fewer than `need_eq` equal keys precede it -- so equal
//      scores go to the lower index and the output is ascending;
//   5. the forced tail (the probe rows) is appended.
// Keys stay in shared memory when they fit, so the score vectors are read
// twice (maxima + keys); otherwise every pass recomputes them from L2.
#include "host.hpp"
#include "rowops.cuh"
#include "sm100.cuh"

namespace spts {

constexpr int TK_THREADS = 1024;
constexpr int TK_ITEMS = 8;
constexpr int TK_SMEM_KEYS = 49152;  // 192 KB of cached keys

__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t b = __float_as_uint(f);
  if (b == 0x80000000u) b = 0u;
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float key_value(uint32_t k) {
  uint32_t b = (k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k;
  return __uint_as_float(b);
}

struct FuseArgs {
  const float *sa;
  const float *sb;
  int mode;
  float wa, wb;
  float ma, mb;  // maxima (MAXNORM_ADD)
};

__device__ __forceinline__ float fused(const FuseArgs &f, int64_t i) {
  const float s = __ldg(f.sa + i);
  if (f.mode == SPTS_FUSE_NONE) return s;
  const float c = __ldg(f.sb + i);
  if (f.mode == SPTS_FUSE_MULTIPLY) return __fmul_rn(s, c);
  const float ta = f.ma > 0.f ? __fmul_rn(f.wa, __fdiv_rn(s, f.ma)) : 0.f;
  const float tb = f.mb > 0.f ? __fmul_rn(f.wb, __fdiv_rn(c, f.mb)) : 0.f;
  return __fadd_rn(ta, tb);
}

// Block-wide exclusive scan of one uint32 per thread (1024 threads).
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t *warp_tot, uint32_t *total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_tot[w] = x;
  __syncthreads();
  if (w == 0) {
    uint32_t t = warp_tot[lane], u = t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      uint32_t y = __shfl_up_sync(0xffffffffu, u, o);
      if (lane >= o) u += y;
    }
    warp_tot[lane] = u - t;  // exclusive prefix of warp totals
    if (lane == 31) *total = u;
  }
  __syncthreads();
  const uint32_t r = warp_tot[w] + x - v;
  __syncthreads();
  return r;
}

template <bool CACHE>
__global__ void __launch_bounds__(TK_THREADS, 1)
    select_topk_kernel(FuseArgs fa, int64_t Nc, int64_t k, int64_t tail, int32_t *__restrict__ idx_out,
                       float *__restrict__ fused_out, float *__restrict__ kth_out, uint32_t *status) {
  extern __shared__ uint32_t keys[];  // CACHE: keys of the first Nc - tail candidates
  __shared__ uint32_t hist[256];
  __shared__ uint32_t warp_tot[32];
  __shared__ float fred[2][32];
  __shared__ uint32_t s_digit, s_krem, s_total;
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int64_t n_free = Nc - tail;
  const int64_t k_free = k - tail;

  // 1. maxima over all Nc candidates
  if (fa.mode == SPTS_FUSE_MAXNORM_ADD) {
    float ma = -INFINITY, mb = -INFINITY;
    for (int64_t i = tid; i < Nc; i += TK_THREADS) {
      ma = fmaxf(ma, __ldg(fa.sa + i));
      mb = fmaxf(mb, __ldg(fa.sb + i));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      ma = fmaxf(ma, __shfl_xor_sync(0xffffffffu, ma, o));
      mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, o));
    }
    if (lane == 0) {
      fred[0][w] = ma;
      fred[1][w] = mb;
    }
    __syncthreads();
    ma = fred[0][0];
    mb = fred[1][0];
    for (int t = 1; t < 32; ++t) {
      ma = fmaxf(ma, fred[0][t]);
      mb = fmaxf(mb, fred[1][t]);
    }
    fa.ma = ma;
    fa.mb = mb;
  }

  // 2. fused scores, keys, fused_out, finiteness check
  for (int64_t i = tid; i < Nc; i += TK_THREADS) {
    const float f = fused(fa, i);
    if (!isfinite(f)) raise_status(status, SPTS_DEV_BADINDEX, 0x71u, static_cast<uint32_t>(i));
    if (fused_out) fused_out[i] = f;
    if (CACHE && i < n_free) keys[i] = order_key(f);
  }
  __syncthreads();

  auto key_at = [&](int64_t i) -> uint32_t {
    if (CACHE) return keys[i];
    return order_key(fused(fa, i));
  };

  // 3. radix select of the k_free-th largest key among [0, n_free)
  uint32_t T = 0xFFFFFFFFu, need_eq = 0;
  if (k_free > 0) {
    uint32_t prefix = 0, mask = 0, krem = static_cast<uint32_t>(k_free);
    for (int shift = 24; shift >= 0; shift -= 8) {
      for (int b = tid; b < 256; b += TK_THREADS) hist[b] = 0;
      __syncthreads();
      for (int64_t i = tid; i < n_free; i += TK_THREADS) {
        const uint32_t key = key_at(i);
        if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
      }
      __syncthreads();
      if (w == 0) {
        // lane l owns bins 255-8l .. 248-8l (descending)
        uint32_t c[8], sum = 0;
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          c[t] = hist[255 - 8 * lane - t];
          sum += c[t];
        }
        uint32_t incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        uint32_t above = incl - sum;  // keys in bins higher than my first bin
        if (above < krem && krem <= incl) {
#pragma unroll
          for (int t = 0; t < 8; ++t) {
            if (above < krem && krem <= above + c[t]) {
              s_digit = static_cast<uint32_t>(255 - 8 * lane - t);
              s_krem = krem - above;
            }
            above += c[t];
          }
        }
      }
      __syncthreads();
      prefix |= s_digit << shift;
      mask |= 255u << shift;
      krem = s_krem;
      __syncthreads();
    }
    T = prefix;
    need_eq = krem;
  }

  // 4. stable compaction in index order
  uint32_t run_gt = 0, run_eq = 0;
  if (k_free > 0) {
    for (int64_t base = 0; base < n_free; base += static_cast<int64_t>(TK_THREADS) * TK_ITEMS) {
      const int64_t i0 = base + static_cast<int64_t>(tid) * TK_ITEMS;
      uint32_t kk[TK_ITEMS];
      uint32_t ngt = 0, neq = 0;
#pragma unroll
      for (int t = 0; t < TK_ITEMS; ++t) {
        const int64_t i = i0 + t;
        kk[t] = (i < n_free) ? key_at(i) : 0u;
        if (i < n_free) {
          ngt += kk[t] > T;
          neq += kk[t] == T;
        }
      }
      const uint32_t packed = ngt | (neq << 16);
      const uint32_t excl = block_excl_scan(packed, warp_tot, &s_total);
      uint32_t gt_before = run_gt + (excl & 0xFFFFu);
      uint32_t eq_before = run_eq + (excl >> 16);
#pragma unroll
      for (int t = 0; t < TK_ITEMS; ++t) {
        const int64_t i = i0 + t;
        if (i >= n_free) break;
        if (kk[t] > T) {
          idx_out[gt_before + min(eq_before, need_eq)] = static_cast<int32_t>(i);
          ++gt_before;
        } else if (kk[t] == T) {
          if (eq_before < need_eq) idx_out[gt_before + eq_before] = static_cast<int32_t>(i);
          ++eq_before;
        }
      }
      run_gt += s_total & 0xFFFFu;
      run_eq += s_total >> 16;
      __syncthreads();
    }
  }

  // 5. forced tail and the threshold
  for (int64_t t = tid; t < tail; t += TK_THREADS) idx_out[k_free + t] = static_cast<int32_t>(n_free + t);
  if (tid == 0 && kth_out) *kth_out = k_free > 0 ? key_value(T) : __uint_as_float(0x7FC00000u);
}

spts_status launch_select_topk(const float *s_a, const float *s_b, int mode, float w_a, float w_b, int64_t Nc,
                               int64_t k, int64_t force_tail, int32_t *idx_out, float *fused_out,
                               float *kth_out, uint32_t *status, cudaStream_t s) {
  FuseArgs fa{s_a, s_b, mode, w_a, w_b, 0.f, 0.f};
  const int64_t n_free = Nc - force_tail;
  if (n_free <= TK_SMEM_KEYS) {
    const size_t smem = static_cast<size_t>(n_free > 0 ? n_free : 1) * sizeof(uint32_t);
    static bool attr = false;
    if (!attr) {
      SPTS_CUDA_TRY(cudaFuncSetAttribute(select_topk_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         TK_SMEM_KEYS * sizeof(uint32_t)));
      attr = true;
    }
    select_topk_kernel<true><<<1, TK_THREADS, smem, s>>>(fa, Nc, k, force_tail, idx_out, fused_out, kth_out,
                                                         status);
    note_launch();
  } else {
    select_topk_kernel<false><<<1, TK_THREADS, 0, s>>>(fa, Nc, k, force_tail, idx_out, fused_out, kth_out,
                                                       status);
    note_launch();
  }
  SPTS_CUDA_TRY(cudaGetLastError());
  return SPTS_OK;
}

}  // namespace spts
