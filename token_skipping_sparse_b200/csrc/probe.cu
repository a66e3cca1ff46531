// probe.cu -- Partial Attention Probing on sm_100a (Fig. 2(a)).
//
// Score of key j: s_j = sum over heads h and probes p of the causal softmax
// weight a[h,p,j].  Two passes over the keys, both on tcgen05:
//   pass 1 (row statistics): per (KV head g, key split) a CTA holds the Q
//     tiles of all of the group's probe rows (up to 4 x 128 rows: 128/G
//     probes x G heads each) and, for every key tile of its range, computes
//     S = Q_u K^T for each row tile u (M = 128 rows, N = 128 keys), keeping
//     each row's running max and sum of exp2 (log2 domain).  A combine kernel
//     merges the partial statistics into max + log2(sum) per row.
//   pass 2 (column sums): per (KV head g, key split) a CTA holds all of the
//     group's probe rows and computes transposed tiles S^T = K Q_u^T (M = 128
//     keys, N = 128 probe rows of chunk u), so each TMEM lane is one key and
//     its score is a per-thread sum over the row: no atomics, fixed order,
//     deterministic.  It writes group_scores[g][j]; a final kernel adds the
//     groups.
// Both passes: warp 0 TMA, warp 1 MMA, two consumer warpgroups (warps 4..7
// and 8..11) that take alternate key tiles, each with two TMEM buffers of 128
// columns, so that one warpgroup's exponentials overlap the other's and the
// MMAs of the next work items.  A K tile is loaded once per CTA and feeds all
// row tiles (pass 1) or column chunks (pass 2).  The grids are one wave: one
// CTA per SM.  All waits are bounded.
#include <climits>

#include "host.hpp"
#include "rowops.cuh"
#include "sm100.cuh"

namespace spts {
namespace {

constexpr int THREADS = 384;
// setmaxnreg split: per SMSP one warp of warpgroup 0 (TMA, MMA, idle) and
// one warp of each consumer warpgroup: 80 + 2 x 208 <= 3 x 168.
constexpr int REG_LOW = 80, REG_HIGH = 208;
constexpr int BKEY = 128;
constexpr int TILE_BYTES = 128 * 128 * 2;  // 128 rows x 128 bf16 as two 64-wide swizzled chunks
constexpr int CHUNK_BYTES = 128 * 64 * 2;
constexpr int MAX_RT = 4;                  // probe rows per group <= 512
constexpr int MAX_SPLITS = 64;
constexpr int MAX_STAGES = 4;
constexpr int SMEM_CAP = 232448;           // dynamic shared memory per CTA on sm_100
constexpr float LOG2E = 1.4426950408889634f;

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Work item (local key tile i, sub-item u) uses TMEM buffer (i & 1) * 2 + (u & 1)
// and consumer warpgroup i & 1.  Uses of that buffer before this item:
__device__ __forceinline__ uint32_t buffer_uses(int i, int u, int nsub) {
  const int per_tile = (nsub - (u & 1) + 1) >> 1;  // sub-items of u's parity per key tile
  return static_cast<uint32_t>((i >> 1) * per_tile + (u >> 1));
}

struct Geo {
  const int32_t *ppos;  // [P] probe positions
  const int32_t *kpos;  // [Nc]
  int P, Nc, Hq, Hkv, G, tq;
  int rows_pad;         // probe rows per group padded to 128
  int n_sub;            // row tiles (pass 1) / column chunks (pass 2) = rows_pad / 128
  int splits;           // key splits (CTAs per group)
  int stages;           // K ring depth
  float scale_log2;
  uint32_t *status;
  uint64_t wait_ns;
};

struct Smem {
  uint8_t *q, *k;
  uint64_t *q_full, *k_full, *k_empty, *s_full, *s_free, *drain;
  uint32_t *tmem_holder;
  volatile int *abort_flag;
  int *ranges;  // [0..MAX_RT) kv_end per row tile, [MAX_RT..2 MAX_RT) mask_from, [2 MAX_RT] kv_end of the group
  float *colv;  // pass 2: per column max + log2(sum)
  int32_t *colp;  // pass 2: per column probe position
};

__device__ __forceinline__ Smem carve_smem(uint8_t *smem_raw, const Geo &p, bool cols) {
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Smem s;
  s.q = smem;
  s.k = smem + p.n_sub * TILE_BYTES;
  uint8_t *tail = s.k + p.stages * TILE_BYTES;
  if (cols) {
    s.colv = reinterpret_cast<float *>(tail);
    s.colp = reinterpret_cast<int32_t *>(tail + MAX_RT * 128 * 4);
    tail += MAX_RT * 128 * 8;
  } else {
    s.colv = nullptr;
    s.colp = nullptr;
  }
  uint64_t *bars = reinterpret_cast<uint64_t *>(tail);
  s.q_full = bars;
  s.k_full = bars + 1;
  s.k_empty = s.k_full + MAX_STAGES;
  s.s_full = s.k_empty + MAX_STAGES;
  s.s_free = s.s_full + 4;
  s.drain = s.s_free + 4;
  s.tmem_holder = reinterpret_cast<uint32_t *>(s.drain + 1);
  s.abort_flag = reinterpret_cast<volatile int *>(s.tmem_holder + 1);
  s.ranges = reinterpret_cast<int *>(s.tmem_holder + 2);
  return s;
}
constexpr size_t BAR_BYTES = (1 + 2 * MAX_STAGES + 4 + 4 + 1) * 8 + 8 + (2 * MAX_RT + 1) * 4;

__device__ __forceinline__ void init_barriers(const Smem &s, const Geo &p) {
  mbar_init(s.q_full, 1);
  for (int st = 0; st < p.stages; ++st) {
    mbar_init(&s.k_full[st], 1);
    mbar_init(&s.k_empty[st], 1);
  }
  for (int b = 0; b < 4; ++b) {
    mbar_init(&s.s_full[b], 1);
    mbar_init(&s.s_free[b], 128);
  }
  mbar_init(s.drain, 1);
  *s.abort_flag = 0;
  fence_mbar_init();
}

// Key tiles [kt0, kt1) of this CTA's split of the group's visible keys.
__device__ __forceinline__ void split_range(int kv_end, int split, int splits, int &kt0, int &kt1) {
  const int n_kt = (kv_end + BKEY - 1) / BKEY;
  const int per = (n_kt + splits - 1) / splits;
  kt0 = min(n_kt, split * per);
  kt1 = min(n_kt, (split + 1) * per);
}

// warp 0: Q tiles of the group once, then the K tiles [kt0, kt0 + n) through the ring.
// Pass 1 wants row tile u as one K-major operand (its two 64-wide chunks
// adjacent); pass 2 wants each 64-wide chunk of all rows as one operand.
__device__ __forceinline__ void producer(const Smem &s, const Geo &p, const CUtensorMap *tmQ, const CUtensorMap *tmK,
                                         int g, int kt0, int n, bool chunk_major) {
  mbar_arrive_expect_tx(s.q_full, p.n_sub * TILE_BYTES);
  for (int u = 0; u < p.n_sub; ++u) {
    uint8_t *d0 = chunk_major ? s.q + u * CHUNK_BYTES : s.q + u * TILE_BYTES;
    uint8_t *d1 = chunk_major ? s.q + (p.n_sub + u) * CHUNK_BYTES : s.q + u * TILE_BYTES + CHUNK_BYTES;
    tma_load_3d(d0, tmQ, s.q_full, 0, g * p.G, u * p.tq);
    tma_load_3d(d1, tmQ, s.q_full, 64, g * p.G, u * p.tq);
  }
  uint32_t issued = 0, par = 0;
  for (int i = 0; i < n; ++i) {
    const int st = i % p.stages;
    const uint32_t ph = (i / p.stages) & 1;
    if (!mbar_wait(&s.k_empty[st], ph ^ 1u, s.abort_flag, p.status, p.wait_ns, 0x31u)) break;
    mbar_arrive_expect_tx(&s.k_full[st], TILE_BYTES);
    const int key0 = (kt0 + i) * BKEY;
    tma_load_3d(s.k + st * TILE_BYTES, tmK, &s.k_full[st], 0, g, key0);
    tma_load_3d(s.k + st * TILE_BYTES + CHUNK_BYTES, tmK, &s.k_full[st], 64, g, key0);
    issued |= 1u << st;
    par = (par & ~(1u << st)) | (ph << st);
  }
  if (*s.abort_flag) {
    mbar_drain(s.q_full, 0, p.status);
    for (int st = 0; st < p.stages; ++st)
      if (issued & (1u << st)) mbar_drain(&s.k_full[st], (par >> st) & 1u, p.status);
  }
}

// warp 1 (the whole warp; one elected lane issues each MMA and commit): for
// each key tile, one 8-MMA group per sub-item into its buffer.
// Pass 1: D = Q_u K^T (A = row tile u, B = K tile).  Pass 2: D = K Q_u^T
// (A = K tile, B = column chunk u of the probe rows).
__device__ __forceinline__ void mma_issuer(const Smem &s, const Geo &p, uint32_t tmem, int n, bool transposed) {
  constexpr uint32_t idesc = idesc_bf16_f32(128, 128, 0, 0);
  bool ok = __all_sync(0xffffffffu, mbar_wait(s.q_full, 0, s.abort_flag, p.status, p.wait_ns, 0x32u));
  tc_fence_after();
  const uint32_t q_addr = smem_u32(s.q);
  for (int i = 0; ok && i < n; ++i) {
    const int st = i % p.stages;
    if (!__all_sync(0xffffffffu,
                    mbar_wait(&s.k_full[st], (i / p.stages) & 1, s.abort_flag, p.status, p.wait_ns, 0x33u)))
      break;
    const uint32_t k_addr = smem_u32(s.k + st * TILE_BYTES);
    for (int u = 0; ok && u < p.n_sub; ++u) {
      const int b = (i & 1) * 2 + (u & 1);
      const uint32_t use = buffer_uses(i, u, p.n_sub);
      if (!__all_sync(0xffffffffu,
                      mbar_wait(&s.s_free[b], (use & 1u) ^ 1u, s.abort_flag, p.status, p.wait_ns, 0x34u))) {
        ok = false;
        break;
      }
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t kc = k_addr + (kk >> 2) * CHUNK_BYTES;
        const uint32_t qc = transposed ? q_addr + ((kk >> 2) * p.n_sub + u) * CHUNK_BYTES
                                       : q_addr + u * TILE_BYTES + (kk >> 2) * CHUNK_BYTES;
        const uint64_t qd = sdesc_k_sw128(qc) + 2 * (kk & 3), kd = sdesc_k_sw128(kc) + 2 * (kk & 3);
        mma_bf16_ss_w(tmem + b * 128, transposed ? kd : qd, transposed ? qd : kd, idesc, kk > 0);
      }
      tc_commit_w(&s.s_full[b]);
    }
    if (ok) tc_commit_w(&s.k_empty[st]);
  }
  tc_commit_w(s.drain);
  mbar_drain(s.drain, 0, p.status);
}

// Loads the 128 fp32 columns of buffer b for this warp's 32 lanes, then
// releases the buffer to the MMA warp.  False when the CTA is aborting.
__device__ __forceinline__ bool take_buffer(const Smem &s, const Geo &p, uint32_t lane_base, int b, uint32_t use,
                                            uint32_t (&xr)[128], uint32_t where) {
  const bool ok = mbar_wait(&s.s_full[b], use & 1u, s.abort_flag, p.status, p.wait_ns, where);
  if (!__all_sync(0xffffffffu, ok)) return false;
  tc_fence_after();
#pragma unroll
  for (int c = 0; c < 4; ++c)
    tmem_ld32(lane_base + b * 128 + c * 32, *reinterpret_cast<uint32_t(*)[32]>(xr + 32 * c));
  tmem_ld_wait();
  tc_fence_before();
  mbar_arrive(&s.s_free[b]);
  return true;
}

__device__ __forceinline__ void search_ranges(const Smem &s, const Geo &p, int n_rt) {
  // warps 4..11: one search each: row tile u's last probe (kv_end) and
  // first probe (mask_from)
  const int w = static_cast<int>(threadIdx.x >> 5) - 4;
  if (w >= 0 && w < 2 * n_rt) {
    const int u = w >> 1;
    const int first = u * p.tq, last = min(first + p.tq, p.P) - 1;
    const int r = warp_upper_bound(p.kpos, p.Nc, p.ppos[(w & 1) ? first : last]);
    if ((threadIdx.x & 31) == 0) s.ranges[(w & 1) ? MAX_RT + u : u] = r;
  }
}

// ------------------------------------------------------------------ pass 1
__global__ void __launch_bounds__(THREADS, 1)
    probe_stats_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ Geo p, float2 *__restrict__ partial) {
  extern __shared__ uint8_t smem_raw[];
  const Smem s = carve_smem(smem_raw, p, false);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int split = blockIdx.x % p.splits;
  const int g = blockIdx.x / p.splits;
  const int n_rt = p.n_sub;

  if (threadIdx.x == 0) init_barriers(s, p);
  if (warp == 1) {
    tmem_alloc(s.tmem_holder, 512);
    tmem_relinquish();
  }
  search_ranges(s, p, n_rt);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s.tmem_holder;
  const int kv_group = s.ranges[n_rt - 1];  // the last row tile sees the most keys
  int kt0, kt1;
  split_range(kv_group, split, p.splits, kt0, kt1);
  const int n = kt1 - kt0;

  if (warp == 0) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(REG_LOW));
    if (lane == 0) producer(s, p, &tmQ, &tmK, g, kt0, n, false);
    __syncwarp();
  } else if (warp == 1) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(REG_LOW));
    mma_issuer(s, p, tmem, n, false);
    __syncwarp();
  } else if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(REG_LOW));  // idle
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(REG_HIGH));
    const int wg = (warp - 4) >> 2;
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    const float c2 = p.scale_log2;
    float m[MAX_RT], l[MAX_RT];
#pragma unroll
    for (int q = 0; q < MAX_RT; ++q) {
      m[q] = -INFINITY;
      l[q] = 0.f;
    }
    bool ok = true;
    for (int i = wg; ok && i < n; i += 2) {
      const int j0 = (kt0 + i) * BKEY;
      for (int u = 0; u < n_rt; ++u) {
        const int b = wg * 2 + (u & 1);
        uint32_t xr[128];
        if (!take_buffer(s, p, lane_base, b, buffer_uses(i, u, n_rt), xr, 0x35u)) {
          ok = false;
          break;
        }
        const int kv_end = s.ranges[u], mask_from = s.ranges[MAX_RT + u];
        if (j0 + BKEY > mask_from || j0 + BKEY > kv_end) {
          const int pr = u * p.tq + r / p.G;
          const int32_t qp = pr < p.P ? p.ppos[pr] : INT_MIN;
#pragma unroll
          for (int c = 0; c < BKEY; ++c) {
            const int key = j0 + c;
            if (!(key < kv_end && __ldg(p.kpos + key) <= qp)) xr[c] = 0xff800000u;  // -inf
          }
        }
        float m8[8];
#pragma unroll
        for (int t = 0; t < 8; ++t) m8[t] = __uint_as_float(xr[t]);
#pragma unroll
        for (int c = 8; c < BKEY; c += 2)
          m8[(c >> 1) & 7] = fmax3(m8[(c >> 1) & 7], __uint_as_float(xr[c]), __uint_as_float(xr[c + 1]));
        const float mt = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                               fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7]))) * c2;
        float mu = m[0], lu = l[0];
#pragma unroll
        for (int q = 1; q < MAX_RT; ++q)
          if (q == u) {
            mu = m[q];
            lu = l[q];
          }
        const float m_new = fmaxf(mu, mt);
        if (m_new == -INFINITY) continue;  // nothing visible yet
        const float neg = -m_new;
        float s8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int c = 0; c < BKEY; ++c) s8[c & 7] += ex2(fmaf(__uint_as_float(xr[c]), c2, neg));
        const float sum = ((s8[0] + s8[1]) + (s8[2] + s8[3])) + ((s8[4] + s8[5]) + (s8[6] + s8[7]));
        lu = (mu == -INFINITY ? 0.f : lu * ex2(mu - m_new)) + sum;
#pragma unroll
        for (int q = 0; q < MAX_RT; ++q)
          if (q == u) {
            m[q] = m_new;
            l[q] = lu;
          }
      }
    }
    if (ok) {
#pragma unroll
      for (int q = 0; q < MAX_RT; ++q)
        if (q < n_rt)
          partial[(static_cast<int64_t>(split * 2 + wg) * p.Hkv + g) * p.rows_pad + q * 128 + r] =
              make_float2(m[q], l[q]);
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// merge the partials: stats[g][row].x = max + log2(sum) in log2 units
__global__ void probe_combine_kernel(const float2 *__restrict__ partial, int parts, int total,
                                     float2 *__restrict__ stats) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= total) return;
  float m = -INFINITY;
  for (int s = 0; s < parts; ++s) m = fmaxf(m, partial[static_cast<int64_t>(s) * total + i].x);
  float l = 0.f;
  if (m != -INFINITY)
    for (int s = 0; s < parts; ++s) {
      const float2 v = partial[static_cast<int64_t>(s) * total + i];
      if (v.x != -INFINITY) l += v.y * ex2(v.x - m);
    }
  // pass 2 weighs key j by 2^(s_j - m - log2 l): fold the normaliser into the exponent
  stats[i] = make_float2(l > 0.f ? m + __log2f(l) : INFINITY, 0.f);
}

// ------------------------------------------------------------------ pass 2
__global__ void __launch_bounds__(THREADS, 1)
    probe_scores_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ Geo p, const float2 *__restrict__ stats, float *__restrict__ group) {
  extern __shared__ uint8_t smem_raw[];
  const Smem s = carve_smem(smem_raw, p, true);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int split = blockIdx.x % p.splits;
  const int g = blockIdx.x / p.splits;
  const int ncol = p.rows_pad;

  for (int c = threadIdx.x; c < MAX_RT * 128; c += THREADS) {
    const int pr = c / p.G;
    const bool live = c < ncol && pr < p.P;
    s.colv[c] = live ? stats[g * ncol + c].x : INFINITY;
    s.colp[c] = live ? p.ppos[pr] : INT_MIN;
  }
  if (threadIdx.x == 0) init_barriers(s, p);
  if (warp == 1) {
    tmem_alloc(s.tmem_holder, 512);
    tmem_relinquish();
  }
  if (warp == 4) {
    const int r = warp_upper_bound(p.kpos, p.Nc, p.ppos[p.P - 1]);
    if (lane == 0) s.ranges[2 * MAX_RT] = r;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s.tmem_holder;
  const int kv_end = s.ranges[2 * MAX_RT];
  int kt0, kt1;
  split_range(kv_end, split, p.splits, kt0, kt1);
  const int n = kt1 - kt0;
  const int32_t ppos_min = p.ppos[0];

  if (warp == 0) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(REG_LOW));
    if (lane == 0) producer(s, p, &tmQ, &tmK, g, kt0, n, true);
    __syncwarp();
  } else if (warp == 1) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(REG_LOW));
    mma_issuer(s, p, tmem, n, true);
    __syncwarp();
  } else if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(REG_LOW));  // idle
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(REG_HIGH));
    const int wg = (warp - 4) >> 2;
    const int quad = warp & 3;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    const float c2 = p.scale_log2;
    bool ok = true;
    for (int i = wg; ok && i < n; i += 2) {
      const int j = (kt0 + i) * BKEY + quad * 32 + lane;
      const bool live = j < kv_end;
      const int32_t kp = live ? __ldg(p.kpos + j) : INT_MAX;
      const bool all_vis = kp <= ppos_min;
      float a4[4] = {0.f, 0.f, 0.f, 0.f};
      for (int u = 0; u < p.n_sub; ++u) {
        const int b = wg * 2 + (u & 1);
        uint32_t xr[128];
        if (!take_buffer(s, p, lane_base, b, buffer_uses(i, u, p.n_sub), xr, 0x45u)) {
          ok = false;
          break;
        }
        const float *cv = s.colv + u * 128;
        if (all_vis) {
#pragma unroll
          for (int t = 0; t < 128; t += 4) {
            const float4 mq = *reinterpret_cast<const float4 *>(cv + t);
            a4[0] += ex2(fmaf(__uint_as_float(xr[t + 0]), c2, -mq.x));
            a4[1] += ex2(fmaf(__uint_as_float(xr[t + 1]), c2, -mq.y));
            a4[2] += ex2(fmaf(__uint_as_float(xr[t + 2]), c2, -mq.z));
            a4[3] += ex2(fmaf(__uint_as_float(xr[t + 3]), c2, -mq.w));
          }
        } else {
          const int32_t *cp = s.colp + u * 128;
#pragma unroll
          for (int t = 0; t < 128; ++t) {
            const float w = ex2(fmaf(__uint_as_float(xr[t]), c2, -cv[t]));
            a4[t & 3] += kp > cp[t] ? 0.f : w;
          }
        }
      }
      if (ok && live) group[static_cast<int64_t>(g) * p.Nc + j] = (a4[0] + a4[1]) + (a4[2] + a4[3]);
    }
    // keys beyond every probe position get no weight
    if (ok && split == p.splits - 1)
      for (int jj = kv_end + (static_cast<int>(threadIdx.x) - 128); jj < p.Nc; jj += THREADS - 128)
        group[static_cast<int64_t>(g) * p.Nc + jj] = 0.f;
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

int rows_pad_of(int P, int G) { return ((P * G + 127) / 128) * 128; }

size_t smem_bytes(int n_sub, int stages, bool cols) {
  return 1024 + static_cast<size_t>(n_sub + stages) * TILE_BYTES + (cols ? MAX_RT * 128 * 8 : 0) + BAR_BYTES;
}
int stages_for(int n_sub, bool cols) {
  int st = MAX_STAGES;
  while (st > 2 && smem_bytes(n_sub, st, cols) > static_cast<size_t>(SMEM_CAP)) --st;
  return st;
}

}  // namespace

size_t probe_bf16_stats_bytes(int P, int Hq, int64_t) {
  // partials of both warpgroups of every split plus the combined statistics;
  // worst case over G: Hkv * rows_pad <= Hq * P + 127 * Hq
  const size_t rows = static_cast<size_t>(Hq) * P + 127 * static_cast<size_t>(Hq);
  return (2 * MAX_SPLITS + 1) * rows * sizeof(float2);
}

spts_status launch_probe_bf16(const void *q, const int32_t *qpos, int P, const void *k, const int32_t *kpos,
                              int64_t Nc, int Hq, int Hkv, float scale, float *group, float *row_stats,
                              uint32_t *status, cudaStream_t s) {
  const int G = Hq / Hkv;
  const int tq = 128 / G;
  const int rows_pad = rows_pad_of(P, G);
  if (rows_pad > MAX_RT * 128) {
    set_error("spts_probe_scores: P * (Hq/Hkv) must be <= 512 on the bf16 path (got %d)", P * G);
    return SPTS_ERR_UNSUPPORTED;
  }
  CUtensorMap tq_map, tk_map;
  {
    uint64_t dims[3] = {128, static_cast<uint64_t>(Hq), static_cast<uint64_t>(P)};
    uint64_t strides[2] = {128 * 2, static_cast<uint64_t>(Hq) * 128 * 2};
    uint32_t box[3] = {64, static_cast<uint32_t>(G), static_cast<uint32_t>(tq)};
    SPTS_TRY(make_tmap(&tq_map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, q, dims, strides, box,
                       CU_TENSOR_MAP_SWIZZLE_128B));
  }
  {
    uint64_t dims[3] = {128, static_cast<uint64_t>(Hkv), static_cast<uint64_t>(Nc)};
    uint64_t strides[2] = {128 * 2, static_cast<uint64_t>(Hkv) * 128 * 2};
    uint32_t box[3] = {64, 1, BKEY};
    SPTS_TRY(make_tmap(&tk_map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, k, dims, strides, box,
                       CU_TENSOR_MAP_SWIZZLE_128B));
  }
  const int n_kt = static_cast<int>((Nc + BKEY - 1) / BKEY);
  Geo geo{};
  geo.ppos = qpos;
  geo.kpos = kpos;
  geo.P = P;
  geo.Nc = static_cast<int>(Nc);
  geo.Hq = Hq;
  geo.Hkv = Hkv;
  geo.G = G;
  geo.tq = tq;
  geo.rows_pad = rows_pad;
  geo.n_sub = rows_pad / 128;
  geo.splits = std::max(1, std::min(std::min(num_sms() / Hkv, MAX_SPLITS), n_kt));
  geo.scale_log2 = scale * LOG2E;
  geo.status = status;
  geo.wait_ns = wait_limit_ns();

  const int parts = 2 * geo.splits;
  float2 *partial = reinterpret_cast<float2 *>(row_stats);
  float2 *stats = partial + static_cast<size_t>(parts) * Hkv * rows_pad;

  Geo g1 = geo;
  g1.stages = stages_for(geo.n_sub, false);
  const size_t sm1 = smem_bytes(geo.n_sub, g1.stages, false);
  SPTS_CUDA_TRY(cudaFuncSetAttribute(probe_stats_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     static_cast<int>(sm1)));
  probe_stats_kernel<<<Hkv * geo.splits, THREADS, sm1, s>>>(tq_map, tk_map, g1, partial);
  note_launch();
  SPTS_CUDA_TRY(cudaGetLastError());
  const int total = Hkv * rows_pad;
  probe_combine_kernel<<<(total + 255) / 256, 256, 0, s>>>(partial, parts, total, stats);
  note_launch();
  SPTS_CUDA_TRY(cudaGetLastError());

  Geo g2 = geo;
  g2.stages = stages_for(geo.n_sub, true);
  const size_t sm2 = smem_bytes(geo.n_sub, g2.stages, true);
  SPTS_CUDA_TRY(cudaFuncSetAttribute(probe_scores_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     static_cast<int>(sm2)));
  probe_scores_kernel<<<Hkv * geo.splits, THREADS, sm2, s>>>(tq_map, tk_map, g2, stats, group);
  note_launch();
  SPTS_CUDA_TRY(cudaGetLastError());
  return SPTS_OK;
}

}  // namespace spts
