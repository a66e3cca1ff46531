// topk.cu -- token selection of SPTS (the informative tokens of Fig. 2(a)/(b)).
//
// One CTA of 1024 threads:
//   1. (MAXNORM_ADD) block maxima of both score vectors over all Nc;
//   2. fused score f per candidate in fp32, one rounding per operation
//      (w_a*(s/max s) + w_b*(c/max c), or s*c, or s), mapped to an
//      order-preserving uint32 key (-0 -> +0);
//   3. MSB-first radix select, digits of 11, 11 and 10 bits, over the first Nc - tail
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
// Above this many free candidates the grid path runs (given scratch).
// Measured alone (MaxNorm-Add, keep 0.3): the grid path takes ~30 us from
// 26K to 131K candidates, one CTA 25 us at 16K, 35 us at 26K, 39 us at 32K
// and 53 us at 48K.
#ifndef TK_GRID_MIN
#define TK_GRID_MIN 20480
#endif

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
  float ma, mb;  // maxima (MAXNORM_ADD) or means (STD_ADD)
  float da, db;  // standard deviations (STD_ADD)
};

// Mean and population standard deviation from fp64 sums, rounded to fp32.
__device__ __forceinline__ void moments(double sum, double sumsq, int64_t n, float *mean, float *sd) {
  const double mu = sum / static_cast<double>(n);
  const double var = fmax(sumsq / static_cast<double>(n) - mu * mu, 0.0);
  *mean = __double2float_rn(mu);
  *sd = __double2float_rn(sqrt(var));
}

__device__ __forceinline__ float fused(const FuseArgs &f, int64_t i) {
  const float s = __ldg(f.sa + i);
  if (f.mode == SPTS_FUSE_NONE) return s;
  const float c = __ldg(f.sb + i);
  if (f.mode == SPTS_FUSE_MULTIPLY) return __fmul_rn(s, c);
  if (f.mode == SPTS_FUSE_STD_ADD) {
    const float ta = f.da > 0.f ? __fmul_rn(f.wa, __fdiv_rn(__fsub_rn(s, f.ma), f.da)) : 0.f;
    const float tb = f.db > 0.f ? __fmul_rn(f.wb, __fdiv_rn(__fsub_rn(c, f.mb), f.db)) : 0.f;
    return __fadd_rn(ta, tb);
  }
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
  __shared__ uint32_t hist[2048];
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

  // 1b. (STD_ADD) fp64 sums of both scores and their squares over all Nc
  if (fa.mode == SPTS_FUSE_STD_ADD) {
    __shared__ double dred[4][32];
    double v[4] = {0.0, 0.0, 0.0, 0.0};
    for (int64_t i = tid; i < Nc; i += TK_THREADS) {
      const double a = __ldg(fa.sa + i), b = __ldg(fa.sb + i);
      v[0] += a;
      v[1] += a * a;
      v[2] += b;
      v[3] += b * b;
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v[q] += __shfl_xor_sync(0xffffffffu, v[q], o);
      if (lane == 0) dred[q][w] = v[q];
    }
    __syncthreads();
    double t[4] = {0.0, 0.0, 0.0, 0.0};
    for (int k2 = 0; k2 < 32; ++k2)
#pragma unroll
      for (int q = 0; q < 4; ++q) t[q] += dred[q][k2];
    moments(t[0], t[1], Nc, &fa.ma, &fa.da);
    moments(t[2], t[3], Nc, &fa.mb, &fa.db);
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

  // 3. radix select of the k_free-th largest key among [0, n_free): digits of
  // 11, 11 and 10 bits from the top.  Scores in a narrow range share the
  // top 8 bits of their keys; taking 3 mantissa bits more into the first
  // digit spreads them over more bins, so fewer threads collide on one
  // shared-memory counter.
  uint32_t T = 0xFFFFFFFFu, need_eq = 0;
  if (k_free > 0) {
    uint32_t prefix = 0, mask = 0, krem = static_cast<uint32_t>(k_free);
#pragma unroll 1
    for (int pass = 0; pass < 3; ++pass) {
      const int bits = pass < 2 ? 11 : 10;
      const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
      const uint32_t nbins = 1u << bits;
      for (int b = tid; b < static_cast<int>(nbins); b += TK_THREADS) hist[b] = 0;
      __syncthreads();
      for (int64_t i = tid; i < n_free; i += TK_THREADS) {
        const uint32_t key = key_at(i);
        if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & (nbins - 1u)], 1u);
      }
      __syncthreads();
      if (w == 0) {
        // lane l owns the bins nbins-1-l*per .. nbins-(l+1)*per (descending)
        const int per = static_cast<int>(nbins) >> 5;
        const int top = static_cast<int>(nbins) - 1 - lane * per;
        uint32_t sum = 0;  // rotated start per lane: the 32 lanes read 32 different banks
        for (int t = 0; t < per; ++t) sum += hist[top - (t + lane) % per];
        uint32_t incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        uint32_t above = incl - sum;  // keys in bins higher than my first bin
        if (above < krem && krem <= incl) {
          for (int t = 0; t < per; ++t) {
            const uint32_t c = hist[top - t];
            if (above < krem && krem <= above + c) {
              s_digit = static_cast<uint32_t>(top - t);
              s_krem = krem - above;
              break;
            }
            above += c;
          }
        }
      }
      __syncthreads();
      prefix |= s_digit << shift;
      mask |= (nbins - 1u) << shift;
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


// ------------------------------------------------------------------ grid path
// For large candidate sets the single CTA above streams every pass from L2
// through one SM.  The grid path spreads the work:
//   topk_prep_kernel      (grid)   zeroes the top-digit histogram; block
//                                  maxima of both scores (MAXNORM_ADD);
//   topk_keys_kernel      (grid)   maxima of the block maxima, fused score,
//                                  key per candidate into the scratch buffer,
//                                  histogram of the top 11 key bits;
//   topk_digit_kernel     (grid, twice)  every CTA finds the bin of the
//                                  (k - tail)-th largest key in the digits
//                                  so far (a block scan of each histogram),
//                                  then histograms the next digit (bits
//                                  [20, 10), then [9, 0)) of its chunk's keys
//                                  that share that prefix;
//   topk_count_kernel     (grid)   the threshold T from the three digits and
//                                  how many keys equal to T are taken (CTA 0
//                                  records them), then per chunk the keys > T
//                                  and == T;
//   topk_write_kernel     (grid)   the counts of the chunks before its own,
//                                  then stable compaction of its chunk; CTA 0
//                                  appends the forced tail.
// The result is identical to the single-CTA path (same keys, same threshold,
// same index order).
constexpr int TG_THREADS = 1024;
constexpr int TG_MAX_CTAS = 256;
constexpr int TG_BINS = 2048;

struct TopkScratch {
  uint32_t *keys;     // [n_free]
  uint32_t *hist;     // [3][TG_BINS]: the histograms of the three digits
  float *maxpart;     // [2][TG_MAX_CTAS]
  double *sumpart;    // [4][TG_MAX_CTAS]: sums of s, s^2, c, c^2 (STD_ADD)
  uint32_t *chunk;    // [2][TG_MAX_CTAS]: per chunk, keys > T and keys == T
  uint32_t *sel;      // [4]: T, need_eq
};

__host__ __device__ inline size_t tg_round(size_t b) { return (b + 255) & ~size_t(255); }

__host__ __device__ inline TopkScratch tg_carve(void *base, int64_t n_free) {
  uint8_t *p = static_cast<uint8_t *>(base);
  TopkScratch t;
  t.keys = reinterpret_cast<uint32_t *>(p);
  p += tg_round(static_cast<size_t>(n_free) * 4);
  t.hist = reinterpret_cast<uint32_t *>(p);
  p += tg_round(3 * TG_BINS * 4);
  t.maxpart = reinterpret_cast<float *>(p);
  p += tg_round(2 * TG_MAX_CTAS * 4);
  t.sumpart = reinterpret_cast<double *>(p);
  p += tg_round(4 * TG_MAX_CTAS * 8);
  t.chunk = reinterpret_cast<uint32_t *>(p);
  p += tg_round(4 * TG_MAX_CTAS * 4);
  t.sel = reinterpret_cast<uint32_t *>(p);
  return t;
}

__global__ void __launch_bounds__(TG_THREADS)
    topk_prep_kernel(FuseArgs fa, int64_t Nc, int64_t chunk, TopkScratch t) {
  __shared__ float red[2][32];
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  for (int b = blockIdx.x * TG_THREADS + tid; b < 3 * TG_BINS; b += gridDim.x * TG_THREADS) t.hist[b] = 0u;
  const int64_t i0 = blockIdx.x * chunk, i1 = min(Nc, i0 + chunk);
  if (fa.mode == SPTS_FUSE_STD_ADD) {
    __shared__ double dred[4][32];
    double v[4] = {0.0, 0.0, 0.0, 0.0};
    for (int64_t i = i0 + tid; i < i1; i += TG_THREADS) {
      const double a = __ldg(fa.sa + i), b = __ldg(fa.sb + i);
      v[0] += a;
      v[1] += a * a;
      v[2] += b;
      v[3] += b * b;
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v[q] += __shfl_xor_sync(0xffffffffu, v[q], o);
      if (lane == 0) dred[q][w] = v[q];
    }
    __syncthreads();
    if (tid < 4) {
      double acc = 0.0;
      for (int k2 = 0; k2 < 32; ++k2) acc += dred[tid][k2];
      t.sumpart[tid * TG_MAX_CTAS + blockIdx.x] = acc;
    }
    return;
  }
  if (fa.mode != SPTS_FUSE_MAXNORM_ADD) return;
  float ma = -INFINITY, mb = -INFINITY;
  for (int64_t i = i0 + tid; i < i1; i += TG_THREADS) {
    ma = fmaxf(ma, __ldg(fa.sa + i));
    mb = fmaxf(mb, __ldg(fa.sb + i));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    ma = fmaxf(ma, __shfl_xor_sync(0xffffffffu, ma, o));
    mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, o));
  }
  if (lane == 0) {
    red[0][w] = ma;
    red[1][w] = mb;
  }
  __syncthreads();
  if (tid == 0) {
    for (int k = 1; k < 32; ++k) {
      ma = fmaxf(ma, red[0][k]);
      mb = fmaxf(mb, red[1][k]);
    }
    t.maxpart[blockIdx.x] = ma;
    t.maxpart[TG_MAX_CTAS + blockIdx.x] = mb;
  }
}


// Adds 1 to h[bin] for every lane of the warp, one shared-memory atomic per
// distinct bin (the scores of a layer crowd into few top-digit bins).
__device__ __forceinline__ void warp_hist_add(uint32_t *h, uint32_t bin, bool active) {
  const uint32_t act = __ballot_sync(0xffffffffu, active);
  if (!active) return;
  const uint32_t peers = __match_any_sync(act, bin);
  if ((threadIdx.x & 31) == __ffs(peers) - 1) atomicAdd(&h[bin], __popc(peers));
}

__global__ void __launch_bounds__(TG_THREADS)
    topk_keys_kernel(FuseArgs fa, int64_t Nc, int64_t n_free, int64_t chunk, int n_cta, TopkScratch t,
                     float *__restrict__ fused_out, uint32_t *status) {
  __shared__ uint32_t h[TG_BINS];
  __shared__ float mx[2];
  const int tid = threadIdx.x;
  if (fa.mode == SPTS_FUSE_MAXNORM_ADD) {
    if (tid < 64) {
      const int which = tid >> 5, lane = tid & 31;
      float m = -INFINITY;
      for (int c = lane; c < n_cta; c += 32) m = fmaxf(m, t.maxpart[which * TG_MAX_CTAS + c]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      if (lane == 0) mx[which] = m;
    }
  }
  __shared__ double sums[4];
  if (fa.mode == SPTS_FUSE_STD_ADD && tid < 4) {
    double acc = 0.0;
    for (int c = 0; c < n_cta; ++c) acc += t.sumpart[tid * TG_MAX_CTAS + c];  // fixed order
    sums[tid] = acc;
  }
  for (int b = tid; b < TG_BINS; b += TG_THREADS) h[b] = 0u;
  __syncthreads();
  if (fa.mode == SPTS_FUSE_MAXNORM_ADD) {
    fa.ma = mx[0];
    fa.mb = mx[1];
  } else if (fa.mode == SPTS_FUSE_STD_ADD) {
    moments(sums[0], sums[1], Nc, &fa.ma, &fa.da);
    moments(sums[2], sums[3], Nc, &fa.mb, &fa.db);
  }
  const int64_t i0 = blockIdx.x * chunk, i1 = min(Nc, i0 + chunk);
  for (int64_t base = i0; base < i1; base += TG_THREADS) {
    const int64_t i = base + tid;
    uint32_t key = 0u;
    bool counted = false;
    if (i < i1) {
      const float f = fused(fa, i);
      if (!isfinite(f)) raise_status(status, SPTS_DEV_BADINDEX, 0x71u, static_cast<uint32_t>(i));
      if (fused_out) fused_out[i] = f;
      if (i < n_free) {
        key = order_key(f);
        t.keys[i] = key;
        counted = true;
      }
    }
    warp_hist_add(h, key >> 21, counted);
  }
  __syncthreads();
  for (int b = tid; b < TG_BINS; b += TG_THREADS)
    if (h[b]) atomicAdd(&t.hist[b], h[b]);
}

// With the bins in descending order, finds the bin holding the krem-th
// largest of the counted keys; *digit = that bin, *krem_out = its rank
// inside the bin.  nb = 1024 or 2048 bins, 1024 threads.
__device__ __forceinline__ void tg_find_bin(const uint32_t *h, int nb, uint32_t krem, uint32_t *warp_tot,
                                            uint32_t *total, uint32_t *digit, uint32_t *krem_out) {
  const int tid = threadIdx.x;
  const int per = nb / TG_THREADS;  // 1 or 2 bins per thread, highest bins first
  uint32_t c0 = h[nb - 1 - tid * per], c1 = per == 2 ? h[nb - 2 - tid * per] : 0u;
  const uint32_t sum = c0 + c1;
  const uint32_t above = block_excl_scan(sum, warp_tot, total);
  if (above < krem && krem <= above + sum) {
    if (krem <= above + c0) {
      *digit = static_cast<uint32_t>(nb - 1 - tid * per);
      *krem_out = krem - above;
    } else {
      *digit = static_cast<uint32_t>(nb - 2 - tid * per);
      *krem_out = krem - above - c0;
    }
  }
  __syncthreads();
}

// The first `ndig` digits (11, 11, 10 bits from the top) of the key of the
// k_free-th largest key, from the histograms in t.hist: prefix and mask of
// those bits and the rank of that key among the keys sharing the prefix.
// Every thread of the CTA gets the same values.
__device__ __forceinline__ void tg_pick(const TopkScratch &t, int ndig, uint32_t k_free, uint32_t *h,
                                        uint32_t *warp_tot, uint32_t *s_total, uint32_t *s_digit, uint32_t *s_krem,
                                        uint32_t &prefix, uint32_t &mask, uint32_t &krem) {
  prefix = 0u;
  mask = 0u;
  krem = k_free;
  for (int d = 0; d < ndig; ++d) {
    const int shift = d == 0 ? 21 : d == 1 ? 10 : 0;
    const int nb = d == 2 ? 1024 : 2048;
    for (int b = threadIdx.x; b < nb; b += TG_THREADS) h[b] = __ldcg(t.hist + d * TG_BINS + b);
    __syncthreads();
    tg_find_bin(h, nb, krem, warp_tot, s_total, s_digit, s_krem);
    prefix |= *s_digit << shift;
    mask |= static_cast<uint32_t>(nb - 1) << shift;
    krem = *s_krem;
    __syncthreads();  // h and the shared results are reused
  }
}

// Digit `dig` (1: bits [20, 10), 2: bits [9, 0)) of the chunk's keys that
// share the threshold's first `dig` digits, added into t.hist[dig].
__global__ void __launch_bounds__(TG_THREADS)
    topk_digit_kernel(int64_t n_free, int64_t k_free, int64_t chunk2, int dig, TopkScratch t) {
  __shared__ uint32_t h[TG_BINS];
  __shared__ uint32_t warp_tot[32];
  __shared__ uint32_t s_total, s_digit, s_krem;
  uint32_t prefix, mask, krem;
  tg_pick(t, dig, static_cast<uint32_t>(k_free), h, warp_tot, &s_total, &s_digit, &s_krem, prefix, mask, krem);
  const int shift = dig == 1 ? 10 : 0;
  const uint32_t nb = dig == 1 ? 2048u : 1024u;
  for (int b = threadIdx.x; b < TG_BINS; b += TG_THREADS) h[b] = 0u;
  __syncthreads();
  const int64_t i0 = blockIdx.x * chunk2, i1 = min(n_free, i0 + chunk2);
  for (int64_t base = i0; base < i1; base += TG_THREADS) {
    const int64_t i = base + threadIdx.x;
    const uint32_t key = i < i1 ? __ldcg(t.keys + i) : 0u;
    warp_hist_add(h, (key >> shift) & (nb - 1u), i < i1 && (key & mask) == prefix);
  }
  __syncthreads();
  for (int b = threadIdx.x; b < static_cast<int>(nb); b += TG_THREADS)
    if (h[b]) atomicAdd(&t.hist[dig * TG_BINS + b], h[b]);
}

// Per chunk: keys > T and == T (chunk c = keys [c chunk2, (c + 1) chunk2)).
__global__ void __launch_bounds__(TG_THREADS)
    topk_count_kernel(int64_t n_free, int64_t k_free, int64_t chunk2, TopkScratch t, float *__restrict__ kth_out) {
  __shared__ uint32_t red[2][32];
  __shared__ uint32_t h[TG_BINS];
  __shared__ uint32_t warp_tot[32];
  __shared__ uint32_t s_total, s_digit, s_krem;
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  uint32_t T = 0xFFFFFFFFu, need_eq = 0u;  // no free pick: no key is above or at T
  if (k_free > 0) {
    uint32_t mask;
    tg_pick(t, 3, static_cast<uint32_t>(k_free), h, warp_tot, &s_total, &s_digit, &s_krem, T, mask, need_eq);
  }
  if (blockIdx.x == 0 && tid == 0) {
    t.sel[0] = T;
    t.sel[1] = need_eq;
    if (kth_out) *kth_out = k_free > 0 ? key_value(T) : __uint_as_float(0x7FC00000u);
  }
  const int64_t i0 = blockIdx.x * chunk2, i1 = min(n_free, i0 + chunk2);
  uint32_t gt = 0, eq = 0;
  for (int64_t i = i0 + tid; i < i1; i += TG_THREADS) {
    const uint32_t key = t.keys[i];
    gt += key > T;
    eq += key == T;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    gt += __shfl_xor_sync(0xffffffffu, gt, o);
    eq += __shfl_xor_sync(0xffffffffu, eq, o);
  }
  if (lane == 0) {
    red[0][w] = gt;
    red[1][w] = eq;
  }
  __syncthreads();
  if (tid == 0) {
    for (int k = 1; k < 32; ++k) {
      gt += red[0][k];
      eq += red[1][k];
    }
    t.chunk[blockIdx.x] = gt;
    t.chunk[TG_MAX_CTAS + blockIdx.x] = eq;
  }
}

constexpr int TG_ITEMS = 2;

__global__ void __launch_bounds__(TG_THREADS)
    topk_write_kernel(int64_t n_free, int64_t k_free, int64_t tail, int64_t chunk2, TopkScratch t,
                      int32_t *__restrict__ idx_out) {
  __shared__ uint32_t warp_tot[32];
  __shared__ uint32_t s_total;
  const int tid = threadIdx.x;
  if (blockIdx.x == 0)
    for (int64_t q = tid; q < tail; q += TG_THREADS) idx_out[k_free + q] = static_cast<int32_t>(n_free + q);
  if (k_free == 0) return;
  const uint32_t T = t.sel[0], need_eq = t.sel[1];
  // keys > T and == T in the chunks before this one
  __shared__ uint32_t s_before[2];
  if (tid < 32) {
    uint32_t g = 0, e = 0;
    for (int c = tid; c < static_cast<int>(blockIdx.x); c += 32) {
      g += t.chunk[c];
      e += t.chunk[TG_MAX_CTAS + c];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      g += __shfl_xor_sync(0xffffffffu, g, o);
      e += __shfl_xor_sync(0xffffffffu, e, o);
    }
    if (tid == 0) {
      s_before[0] = g;
      s_before[1] = e;
    }
  }
  __syncthreads();
  uint32_t run_gt = s_before[0], run_eq = s_before[1];
  const int64_t i0 = blockIdx.x * chunk2, i1 = min(n_free, i0 + chunk2);
  for (int64_t base = i0; base < i1; base += static_cast<int64_t>(TG_THREADS) * TG_ITEMS) {
    const int64_t j0 = base + static_cast<int64_t>(tid) * TG_ITEMS;
    uint32_t kk[TG_ITEMS];
    uint32_t ngt = 0, neq = 0;
#pragma unroll
    for (int q = 0; q < TG_ITEMS; ++q) {
      const int64_t i = j0 + q;
      kk[q] = i < i1 ? t.keys[i] : 0u;
      if (i < i1) {
        ngt += kk[q] > T;
        neq += kk[q] == T;
      }
    }
    const uint32_t excl = block_excl_scan(ngt | (neq << 16), warp_tot, &s_total);
    uint32_t gt_before = run_gt + (excl & 0xFFFFu);
    uint32_t eq_before = run_eq + (excl >> 16);
#pragma unroll
    for (int q = 0; q < TG_ITEMS; ++q) {
      const int64_t i = j0 + q;
      if (i >= i1) break;
      if (kk[q] > T) {
        idx_out[gt_before + min(eq_before, need_eq)] = static_cast<int32_t>(i);
        ++gt_before;
      } else if (kk[q] == T) {
        if (eq_before < need_eq) idx_out[gt_before + eq_before] = static_cast<int32_t>(i);
        ++eq_before;
      }
    }
    run_gt += s_total & 0xFFFFu;
    run_eq += s_total >> 16;
    __syncthreads();
  }
}

size_t topk_scratch_bytes(int64_t Nc) {
  return tg_round(static_cast<size_t>(Nc > 0 ? Nc : 1) * 4) + tg_round(3 * TG_BINS * 4) + tg_round(2 * TG_MAX_CTAS * 4) +
         tg_round(4 * TG_MAX_CTAS * 8) + tg_round(4 * TG_MAX_CTAS * 4) + 256;
}

spts_status launch_select_topk(const float *s_a, const float *s_b, int mode, float w_a, float w_b, int64_t Nc,
                               int64_t k, int64_t force_tail, int32_t *idx_out, float *fused_out,
                               float *kth_out, uint32_t *status, void *scratch, cudaStream_t s) {
  FuseArgs fa{s_a, s_b, mode, w_a, w_b, 0.f, 0.f, 0.f, 0.f};
  const int64_t n_free = Nc - force_tail;
  if (scratch != nullptr && n_free > TK_GRID_MIN) {
    const TopkScratch t = tg_carve(scratch, n_free);
    const int64_t want = (Nc + TG_THREADS - 1) / TG_THREADS;
    const int n_cta = static_cast<int>(std::min<int64_t>(std::min(num_sms(), TG_MAX_CTAS), want));
    const int64_t chunk = (Nc + n_cta - 1) / n_cta;
    const int64_t chunk2 = (n_free + n_cta - 1) / n_cta;
    topk_prep_kernel<<<n_cta, TG_THREADS, 0, s>>>(fa, Nc, chunk, t);
    note_launch();
    topk_keys_kernel<<<n_cta, TG_THREADS, 0, s>>>(fa, Nc, n_free, chunk, n_cta, t, fused_out, status);
    note_launch();
    if (k > force_tail)
      for (int dig = 1; dig <= 2; ++dig) {
        topk_digit_kernel<<<n_cta, TG_THREADS, 0, s>>>(n_free, k - force_tail, chunk2, dig, t);
        note_launch();
      }
    topk_count_kernel<<<n_cta, TG_THREADS, 0, s>>>(n_free, k - force_tail, chunk2, t, kth_out);
    note_launch();
    topk_write_kernel<<<n_cta, TG_THREADS, 0, s>>>(n_free, k - force_tail, force_tail, chunk2, t, idx_out);
    note_launch();
    SPTS_CUDA_TRY(cudaGetLastError());
    return SPTS_OK;
  }
  if (n_free <= TK_SMEM_KEYS) {
    const size_t smem = static_cast<size_t>(n_free > 0 ? n_free : 1) * sizeof(uint32_t);
    // the attribute is per device: set it on every call (a few microseconds of host time)
    SPTS_CUDA_TRY(cudaFuncSetAttribute(select_topk_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       TK_SMEM_KEYS * sizeof(uint32_t)));
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

spts_status preload_select_topk() {
  cudaFuncAttributes a;
  SPTS_CUDA_TRY(cudaFuncGetAttributes(&a, select_topk_kernel<true>));
  SPTS_CUDA_TRY(cudaFuncGetAttributes(&a, select_topk_kernel<false>));
  return SPTS_OK;
}

size_t select_sequential_scratch_bytes(int64_t Nc) {
  const size_t n = static_cast<size_t>(Nc > 0 ? Nc : 1) * 4;
  return 3 * tg_round(n) + tg_round(topk_scratch_bytes(Nc));
}

// Sequential Select (Table D; reading): the pool = top-k_pool by s_a (tail
// forced), then the top-k by s_b inside the pool (tail forced again), as
// candidate indices ascending.  Three kernels of this file and two gathers.
spts_status launch_select_sequential(const float *s_a, const float *s_b, int64_t Nc, int64_t k_pool, int64_t k,
                                     int64_t force_tail, int32_t *idx_out, void *scratch, uint32_t *status,
                                     cudaStream_t s) {
  const size_t n = static_cast<size_t>(Nc > 0 ? Nc : 1) * 4;
  uint8_t *p = static_cast<uint8_t *>(scratch);
  int32_t *pool = reinterpret_cast<int32_t *>(p);
  float *b_pool = reinterpret_cast<float *>(p + tg_round(n));
  int32_t *local = reinterpret_cast<int32_t *>(p + 2 * tg_round(n));
  void *tk = p + 3 * tg_round(n);
  SPTS_TRY(launch_select_topk(s_a, nullptr, SPTS_FUSE_NONE, 0.f, 0.f, Nc, k_pool, force_tail, pool, nullptr,
                              nullptr, status, tk, s));
  SPTS_TRY(launch_gather_i32(reinterpret_cast<const int32_t *>(s_b), pool, k_pool,
                             reinterpret_cast<int32_t *>(b_pool), s));
  SPTS_TRY(launch_select_topk(b_pool, nullptr, SPTS_FUSE_NONE, 0.f, 0.f, k_pool, k, force_tail, local, nullptr,
                              nullptr, status, tk, s));
  return launch_gather_i32(pool, local, k, idx_out, s);
}

}  // namespace spts
