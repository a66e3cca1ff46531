// probe.cu -- Partial Attention Probing on sm_100a (Fig. 2(a)).
//
// Score of key j: s_j = sum over heads h and probes p of the causal softmax
// weight a[h,p,j].  Two passes over the keys, both on tcgen05:
//   pass 1 (row statistics): per (KV head g, tile of 128 probe rows, key
//     split) a CTA computes S = Q K^T for its key range (M = 128 rows =
//     128/G probes x G heads, N = 128 keys) and keeps each row's running max
//     and sum of exp2 (log2 domain).  A combine kernel merges the splits into
//     (max, 1/sum) per row.
//   pass 2 (column sums): per (KV head g, key chunk) a CTA holds all of the
//     group's probe rows in shared memory and computes the transposed tile
//     S^T = K Q^T (M = 128 keys, N = probe rows), so each TMEM lane is one
//     key and its score is a per-thread sum over the row: no atomics, fixed
//     order, deterministic.  It writes group_scores[g][j]; a final kernel
//     adds the groups.
// Warp roles as in the other kernels: warp 0 TMA, warp 1 MMA, warps 2..5
// consume the accumulators.  All waits are bounded.
#include <climits>

#include "host.hpp"
#include "rowops.cuh"
#include "sm100.cuh"

namespace spts {
namespace {

constexpr int THREADS = 192;
constexpr int BKEY = 128;
constexpr int TILE_BYTES = 128 * 128 * 2;
constexpr int CHUNK_BYTES = 128 * 64 * 2;
constexpr int MAX_SPLITS = 64;
constexpr float LOG2E = 1.4426950408889634f;

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ int upper_bound(const int32_t *a, int n, int32_t v) {
  int lo = 0, hi = n;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (a[mid] <= v) lo = mid + 1;
    else hi = mid;
  }
  return lo;
}

struct Geo {
  const int32_t *ppos;  // [P] probe positions
  const int32_t *kpos;  // [Nc]
  int P, Nc, Hq, Hkv, G, tq;
  int rows_pad;         // probe rows per group padded to 128
  float scale_log2;
  uint32_t *status;
  uint64_t wait_ns;
};

// ------------------------------------------------------------------ pass 1
constexpr int P1_STAGES = 3;
constexpr int P1_OFF_Q = 0;
constexpr int P1_OFF_K = TILE_BYTES;
constexpr int P1_OFF_BAR = P1_OFF_K + P1_STAGES * TILE_BYTES;
constexpr size_t P1_SMEM = 1024 + P1_OFF_BAR + 256;

__global__ void __launch_bounds__(THREADS, 1)
    probe_stats_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ Geo p, int n_rt, int splits, float2 *__restrict__ partial) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sQ = smem + P1_OFF_Q;
  uint8_t *sK = smem + P1_OFF_K;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + P1_OFF_BAR);
  uint64_t *q_full = bars, *k_full = bars + 1, *k_empty = bars + 1 + P1_STAGES, *s_full = bars + 1 + 2 * P1_STAGES,
           *s_free = s_full + 2, *drain = s_free + 2;
  uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(drain + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);
  int *s_range = reinterpret_cast<int *>(tmem_holder + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int split = blockIdx.x % splits;
  const int rt = (blockIdx.x / splits) % n_rt;
  const int g = blockIdx.x / (splits * n_rt);
  const int p0 = rt * p.tq;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < P1_STAGES; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&s_free[b], 128);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    const int last = min(p0 + p.tq, p.P) - 1;
    const int kv_end = upper_bound(p.kpos, p.Nc, p.ppos[last]);
    const int n_kt = (kv_end + BKEY - 1) / BKEY;
    const int per = (n_kt + splits - 1) / splits;
    s_range[0] = min(n_kt, split * per);
    s_range[1] = min(n_kt, (split + 1) * per);
    s_range[2] = kv_end;
    s_range[3] = upper_bound(p.kpos, p.Nc, p.ppos[p0]);
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const int kt0 = s_range[0], kt1 = s_range[1], kv_end = s_range[2], mask_from = s_range[3];
  const int n = kt1 - kt0;

  if (warp == 0) {
    if (lane == 0) {
      mbar_arrive_expect_tx(q_full, TILE_BYTES);
      tma_load_3d(sQ, &tmQ, q_full, 0, g * p.G, p0);
      tma_load_3d(sQ + CHUNK_BYTES, &tmQ, q_full, 64, g * p.G, p0);
      uint32_t issued = 0, par = 0;
      for (int i = 0; i < n; ++i) {
        const int st = i % P1_STAGES;
        const uint32_t ph = (i / P1_STAGES) & 1;
        if (!mbar_wait(&k_empty[st], ph ^ 1u, abort_flag, p.status, p.wait_ns, 0x31u)) break;
        mbar_arrive_expect_tx(&k_full[st], TILE_BYTES);
        const int key0 = (kt0 + i) * BKEY;
        tma_load_3d(sK + st * TILE_BYTES, &tmK, &k_full[st], 0, g, key0);
        tma_load_3d(sK + st * TILE_BYTES + CHUNK_BYTES, &tmK, &k_full[st], 64, g, key0);
        issued |= 1u << st;
        par = (par & ~(1u << st)) | (ph << st);
      }
      if (*abort_flag) {
        mbar_drain(q_full, 0, p.status);
        for (int st = 0; st < P1_STAGES; ++st)
          if (issued & (1u << st)) mbar_drain(&k_full[st], (par >> st) & 1u, p.status);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, BKEY, 0, 0);
      bool ok = mbar_wait(q_full, 0, abort_flag, p.status, p.wait_ns, 0x32u);
      tc_fence_after();
      const uint32_t q_addr = smem_u32(sQ);
      for (int i = 0; ok && i < n; ++i) {
        const int st = i % P1_STAGES, b = i & 1;
        if (!mbar_wait(&s_free[b], ((i >> 1) & 1) ^ 1u, abort_flag, p.status, p.wait_ns, 0x33u)) break;
        if (!mbar_wait(&k_full[st], (i / P1_STAGES) & 1, abort_flag, p.status, p.wait_ns, 0x34u)) break;
        tc_fence_after();
        const uint32_t k_addr = smem_u32(sK + st * TILE_BYTES);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16_ss(tmem + b * BKEY, sdesc_k_sw128(q_addr + (kk >> 2) * CHUNK_BYTES) + 2 * (kk & 3),
                      sdesc_k_sw128(k_addr + (kk >> 2) * CHUNK_BYTES) + 2 * (kk & 3), idesc, kk > 0);
        tc_commit(&k_empty[st]);
        tc_commit(&s_full[b]);
      }
      tc_commit(drain);
      mbar_drain(drain, 0, p.status);
    }
    __syncwarp();
  } else {
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const int pr = p0 + r / p.G;
    const bool valid = pr < p.P;
    const int32_t qp = valid ? p.ppos[pr] : INT_MIN;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int i = 0; i < n; ++i) {
      const int b = i & 1;
      ok = mbar_wait(&s_full[b], (i >> 1) & 1, abort_flag, p.status, p.wait_ns, 0x35u);
      if (!__all_sync(0xffffffffu, ok)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t xr[BKEY];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(lane_base + b * BKEY + c * 32, *reinterpret_cast<uint32_t(*)[32]>(xr + 32 * c));
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(&s_free[b]);
      const int j0 = (kt0 + i) * BKEY;
      const bool need_mask = (j0 + BKEY > mask_from) || (j0 + BKEY > kv_end);
      float x[BKEY], m8[8];
#pragma unroll
      for (int t = 0; t < 8; ++t) m8[t] = -INFINITY;
#pragma unroll
      for (int c = 0; c < BKEY; ++c) {
        float v = __uint_as_float(xr[c]) * p.scale_log2;
        if (need_mask) {
          const int key = j0 + c;
          if (!(key < kv_end && __ldg(p.kpos + key) <= qp)) v = -INFINITY;
        }
        x[c] = v;
        m8[c & 7] = fmaxf(m8[c & 7], v);
      }
      const float mt =
          fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])), fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
      const float m_new = fmaxf(m, mt);
      if (m_new == -INFINITY) continue;
      float s8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c = 0; c < BKEY; ++c) s8[c & 7] += ex2(x[c] - m_new);
      const float sum = ((s8[0] + s8[1]) + (s8[2] + s8[3])) + ((s8[4] + s8[5]) + (s8[6] + s8[7]));
      l = (m == -INFINITY ? 0.f : l * ex2(m - m_new)) + sum;
      m = m_new;
    }
    if (ok) partial[(static_cast<int64_t>(split) * p.Hkv + g) * p.rows_pad + rt * 128 + r] = make_float2(m, l);
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

// merge the splits: stats[g][row].x = max + log2(sum) in log2 units
__global__ void probe_combine_kernel(const float2 *__restrict__ partial, int splits, int total,
                                     float2 *__restrict__ stats) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= total) return;
  float m = -INFINITY;
  for (int s = 0; s < splits; ++s) m = fmaxf(m, partial[static_cast<int64_t>(s) * total + i].x);
  float l = 0.f;
  if (m != -INFINITY)
    for (int s = 0; s < splits; ++s) {
      const float2 v = partial[static_cast<int64_t>(s) * total + i];
      if (v.x != -INFINITY) l += v.y * ex2(v.x - m);
    }
  // pass 2 weighs key j by 2^(s_j - m - log2 l): fold the normaliser into the exponent
  stats[i] = make_float2(l > 0.f ? m + __log2f(l) : INFINITY, 0.f);
}

// ------------------------------------------------------------------ pass 2
constexpr int P2_STAGES = 2;
constexpr int P2_MAX_ROWS = 512;

__global__ void __launch_bounds__(THREADS, 1)
    probe_scores_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ Geo p, int chunks, const float2 *__restrict__ stats,
                        float *__restrict__ group) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int ncol = p.rows_pad;                 // probe rows of this group (padded), <= 512
  const int q_tiles = ncol / 128;
  uint8_t *sQ = smem;                          // q_tiles x 32 KB: rows [ncol] as 64-wide chunks per tile
  uint8_t *sK = smem + q_tiles * TILE_BYTES;   // P2_STAGES x 32 KB
  float *smm = reinterpret_cast<float *>(sK + P2_STAGES * TILE_BYTES);   // per column: max + log2(sum)
  int32_t *scol = reinterpret_cast<int32_t *>(smm + P2_MAX_ROWS);      // per column: probe position
  uint64_t *bars = reinterpret_cast<uint64_t *>(scol + P2_MAX_ROWS);
  uint64_t *q_full = bars, *k_full = bars + 1, *k_empty = bars + 1 + P2_STAGES, *s_full = bars + 1 + 2 * P2_STAGES,
           *s_free = s_full + 2, *drain = s_free + 2;
  uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(drain + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);
  int *s_range = reinterpret_cast<int *>(tmem_holder + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int chunk = blockIdx.x % chunks;
  const int g = blockIdx.x / chunks;
  // the probe rows are processed in chunks of CW columns, one TMEM buffer each
  const int CW = (ncol % 256 == 0) ? 256 : 128;
  const int nch = ncol / CW;
  const uint32_t tmem_cols = 512;

  for (int c = threadIdx.x; c < P2_MAX_ROWS; c += THREADS) {
    const int pr = c / p.G;
    const bool live = c < ncol && pr < p.P;
    smm[c] = live ? stats[g * ncol + c].x : INFINITY;
    scol[c] = live ? p.ppos[pr] : INT_MIN;
  }
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < P2_STAGES; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&s_free[b], 128);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    const int kv_end = upper_bound(p.kpos, p.Nc, p.ppos[p.P - 1]);
    const int n_kt = (kv_end + BKEY - 1) / BKEY;
    const int per = (n_kt + chunks - 1) / chunks;
    s_range[0] = min(n_kt, chunk * per);
    s_range[1] = min(n_kt, (chunk + 1) * per);
    s_range[2] = kv_end;
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const int kt0 = s_range[0], kt1 = s_range[1], kv_end = s_range[2];
  const int n = kt1 - kt0;
  const int32_t ppos_min = p.ppos[0];

  if (warp == 0) {
    if (lane == 0) {
      mbar_arrive_expect_tx(q_full, q_tiles * TILE_BYTES);
      for (int t = 0; t < q_tiles; ++t) {
        // chunk c of every probe row lives at sQ + c*(q_tiles*16KB) + t*16KB, so each
        // 64-wide chunk is one K-major operand of ncol rows
        tma_load_3d(sQ + t * CHUNK_BYTES, &tmQ, q_full, 0, g * p.G, t * p.tq);
        tma_load_3d(sQ + q_tiles * CHUNK_BYTES + t * CHUNK_BYTES, &tmQ, q_full, 64, g * p.G, t * p.tq);
      }
      uint32_t issued = 0, par = 0;
      for (int i = 0; i < n; ++i) {
        const int st = i % P2_STAGES;
        const uint32_t ph = (i / P2_STAGES) & 1;
        if (!mbar_wait(&k_empty[st], ph ^ 1u, abort_flag, p.status, p.wait_ns, 0x41u)) break;
        mbar_arrive_expect_tx(&k_full[st], TILE_BYTES);
        const int key0 = (kt0 + i) * BKEY;
        tma_load_3d(sK + st * TILE_BYTES, &tmK, &k_full[st], 0, g, key0);
        tma_load_3d(sK + st * TILE_BYTES + CHUNK_BYTES, &tmK, &k_full[st], 64, g, key0);
        issued |= 1u << st;
        par = (par & ~(1u << st)) | (ph << st);
      }
      if (*abort_flag) {
        mbar_drain(q_full, 0, p.status);
        for (int st = 0; st < P2_STAGES; ++st)
          if (issued & (1u << st)) mbar_drain(&k_full[st], (par >> st) & 1u, p.status);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(128, CW, 0, 0);
      bool ok = mbar_wait(q_full, 0, abort_flag, p.status, p.wait_ns, 0x42u);
      tc_fence_after();
      // work item it = (key tile it / nch, column chunk it % nch) into TMEM buffer it % 2
      for (int it = 0; ok && it < n * nch; ++it) {
        const int i = it / nch, h = it % nch;
        const int st = i % P2_STAGES;
        const int b = it & 1;
        if (!mbar_wait(&s_free[b], ((it >> 1) & 1) ^ 1u, abort_flag, p.status, p.wait_ns, 0x43u)) break;
        if (h == 0 && !mbar_wait(&k_full[st], (i / P2_STAGES) & 1, abort_flag, p.status, p.wait_ns, 0x44u)) break;
        tc_fence_after();
        const uint32_t k_addr = smem_u32(sK + st * TILE_BYTES);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t a = sdesc_k_sw128(k_addr + (kk >> 2) * CHUNK_BYTES) + 2 * (kk & 3);
          const uint32_t q_addr = smem_u32(sQ + (kk >> 2) * q_tiles * CHUNK_BYTES + h * (CW / 128) * CHUNK_BYTES);
          mma_bf16_ss(tmem + b * CW, a, sdesc_k_sw128(q_addr) + 2 * (kk & 3), idesc, kk > 0);
        }
        if (h == nch - 1) tc_commit(&k_empty[st]);
        tc_commit(&s_full[b]);
      }
      tc_commit(drain);
      mbar_drain(drain, 0, p.status);
    }
    __syncwarp();
  } else {
    const int quad = warp & 3;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    bool ok = true;
    float acc = 0.f;
    for (int it = 0; it < n * nch; ++it) {
      const int i = it / nch, h = it % nch;
      const int b = it & 1;
      ok = mbar_wait(&s_full[b], (it >> 1) & 1, abort_flag, p.status, p.wait_ns, 0x45u);
      if (!__all_sync(0xffffffffu, ok)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int j = (kt0 + i) * BKEY + quad * 32 + lane;
      const bool live = j < kv_end;
      const int32_t kp = live ? __ldg(p.kpos + j) : INT_MAX;
      const bool all_vis = kp <= ppos_min;
      if (h == 0) acc = 0.f;
      float a4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 1
      for (int c0 = 0; c0 < CW; c0 += 32) {
        uint32_t xr[32];
        tmem_ld32(lane_base + b * CW + c0, xr);
        tmem_ld_wait();
        const float *mmc = smm + h * CW + c0;
#pragma unroll
        for (int t = 0; t < 32; t += 4) {
          const float4 mq = *reinterpret_cast<const float4 *>(mmc + t);
          const float mv[4] = {mq.x, mq.y, mq.z, mq.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            float w = ex2(fmaf(__uint_as_float(xr[t + e]), p.scale_log2, -mv[e]));
            if (!all_vis && kp > scol[h * CW + c0 + t + e]) w = 0.f;
            a4[e] += w;
          }
        }
      }
      acc += (a4[0] + a4[1]) + (a4[2] + a4[3]);
      tc_fence_before();
      mbar_arrive(&s_free[b]);
      if (h == nch - 1 && live) group[static_cast<int64_t>(g) * p.Nc + j] = acc;
    }
    // keys beyond every probe position get no weight
    if (ok) {
      const int first = kv_end;
      for (int jj = first + (threadIdx.x - 64); jj < p.Nc && chunk == chunks - 1; jj += 128)
        group[static_cast<int64_t>(g) * p.Nc + jj] = 0.f;
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, tmem_cols);
  }
}

int rows_pad_of(int P, int G) { return ((P * G + 127) / 128) * 128; }

}  // namespace

size_t probe_bf16_stats_bytes(int P, int Hq, int64_t) {
  // worst case over G: Hkv * rows_pad <= Hq * P + 127 * Hq
  const size_t rows = static_cast<size_t>(Hq) * P + 127 * static_cast<size_t>(Hq);
  return (MAX_SPLITS + 1) * rows * sizeof(float2);
}

spts_status launch_probe_bf16(const void *q, const int32_t *qpos, int P, const void *k, const int32_t *kpos,
                              int64_t Nc, int Hq, int Hkv, float scale, float *group, float *row_stats,
                              uint32_t *status, cudaStream_t s) {
  const int G = Hq / Hkv;
  const int tq = 128 / G;
  const int rows_pad = rows_pad_of(P, G);
  if (rows_pad > P2_MAX_ROWS) {
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
  geo.scale_log2 = scale * LOG2E;
  geo.status = status;
  geo.wait_ns = wait_limit_ns();

  const int n_rt = rows_pad / 128;
  const int n_kt = static_cast<int>((Nc + BKEY - 1) / BKEY);
  int splits = (2 * num_sms() + n_rt * Hkv - 1) / (n_rt * Hkv);
  splits = std::max(1, std::min(std::min(splits, MAX_SPLITS), n_kt));
  float2 *partial = reinterpret_cast<float2 *>(row_stats);
  float2 *stats = partial + static_cast<size_t>(splits) * Hkv * rows_pad;

  SPTS_CUDA_TRY(cudaFuncSetAttribute(probe_stats_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     static_cast<int>(P1_SMEM)));
  probe_stats_kernel<<<n_rt * Hkv * splits, THREADS, P1_SMEM, s>>>(tq_map, tk_map, geo, n_rt, splits, partial);
  note_launch();
  SPTS_CUDA_TRY(cudaGetLastError());
  const int total = Hkv * rows_pad;
  probe_combine_kernel<<<(total + 255) / 256, 256, 0, s>>>(partial, splits, total, stats);
  note_launch();
  SPTS_CUDA_TRY(cudaGetLastError());

  const size_t p2_smem = 1024 + static_cast<size_t>(rows_pad / 128) * TILE_BYTES + P2_STAGES * TILE_BYTES +
                         P2_MAX_ROWS * (sizeof(float2) + sizeof(int32_t)) + 256;
  int chunks = (2 * num_sms() + Hkv - 1) / Hkv;
  chunks = std::max(1, std::min(chunks, n_kt));
  SPTS_CUDA_TRY(cudaFuncSetAttribute(probe_scores_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     static_cast<int>(p2_smem)));
  probe_scores_kernel<<<Hkv * chunks, THREADS, p2_smem, s>>>(tq_map, tk_map, geo, chunks, stats, group);
  note_launch();
  SPTS_CUDA_TRY(cudaGetLastError());
  return SPTS_OK;
}

}  // namespace spts
