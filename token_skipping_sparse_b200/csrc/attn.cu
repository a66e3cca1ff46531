// attn.cu -- reduced GQA attention of SPTS on sm_100a (Fig. 2(a): the
// informative tokens attend to every candidate key, causally by original
// position).
//
// One CTA per (Q tile, KV head).  A Q tile packs 128/G selected tokens x the
// G query heads that share KV head g (G = Hq/Hkv), so every K/V tile loaded
// serves all G heads in one M=128 MMA.
//   warp 0      TMA: the Q tile once, then K and V tiles of 128 keys into a
//               3-stage ring (128-byte swizzle);
//   warp 1      MMA: S = Q K^T into one of two TMEM buffers (M=128, N=128,
//               K=128), then O += P V with P read from TMEM (the softmax
//               writes it over the S values it consumed) and V an MN-major
//               shared-memory operand, into a third TMEM region;
//   warps 2..5  softmax, one thread per Q row: tcgen05.ld of its S row,
//               causal mask (only on tiles that cross the diagonal), row max
//               with independent accumulators, lazy rescaling of O in TMEM
//               (only when the running max grows by more than 2^8), exp2 with
//               the scale folded into one FFMA, bf16 P stored back to TMEM
//               with tcgen05.st; at the end O / l -> bf16.
// Keeping P in TMEM takes it off the shared-memory path: per key tile the
// shared memory then serves only the K and V tiles (TMA in, MMA out).
// The key loop stops at the last key visible to the tile's latest query, and
// tiles are launched latest-first so the long ones start early.
// All barrier waits are bounded (see sm100.cuh).
#include <climits>

#include "host.hpp"
#include "rowops.cuh"
#include "sm100.cuh"

namespace spts {
namespace {

constexpr int THREADS = 192;
constexpr int BKV = 128;
constexpr int KV_STAGES = 3;
constexpr int TILE_BYTES = 128 * 128 * 2;  // 32 KB: 128 rows x 128 bf16, as two 64-wide swizzled chunks
constexpr int CHUNK_BYTES = 128 * 64 * 2;  // 16 KB
constexpr int OFF_Q = 0;
constexpr int OFF_K = OFF_Q + TILE_BYTES;               // KV_STAGES stages
constexpr int OFF_V = OFF_K + KV_STAGES * TILE_BYTES;   // KV_STAGES stages
constexpr int OFF_BAR = OFF_V + KV_STAGES * TILE_BYTES;
constexpr size_t SMEM_BYTES = OFF_BAR + 256;
constexpr uint32_t TMEM_COLS = 512;  // S/P buffers [0,128) and [128,256), O [256,384)
constexpr float RESCALE_THRESHOLD = 8.0f;  // log2 units

struct Params {
  const int32_t *qpos;
  const int32_t *kpos;
  __nv_bfloat16 *o;
  int m, Nc, Hq, Hkv, G, tq, n_qtiles;
  float scale_log2;
  uint32_t *status;
  uint64_t wait_ns;
};

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

__global__ void __launch_bounds__(THREADS, 1)
    attention_bf16_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                          const __grid_constant__ CUtensorMap tmV, const __grid_constant__ Params p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t *sQ = smem + OFF_Q;
  uint8_t *sK = smem + OFF_K;
  uint8_t *sV = smem + OFF_V;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
  uint64_t *q_full = bars + 0, *k_full = bars + 1, *v_full = k_full + KV_STAGES, *kv_empty = v_full + KV_STAGES,
           *s_full = kv_empty + KV_STAGES, *p_ready = s_full + 2, *p_free = p_ready + 2, *drain = p_free + 2;
  uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(drain + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);
  int *s_range = reinterpret_cast<int *>(tmem_holder + 2);  // kv_end, mask_from

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = p.n_qtiles - 1 - static_cast<int>(blockIdx.x) / p.Hkv;
  const int g = static_cast<int>(blockIdx.x) % p.Hkv;
  const int t0 = qt * p.tq;

  // The swizzled operand layouts need a 1024-byte aligned base.
  if (smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0) raise_status(p.status, SPTS_DEV_BADINDEX, 0x2Fu, smem_u32(smem));
    return;
  }
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < KV_STAGES; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&p_ready[s], 128);
      mbar_init(&p_free[s], 1);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    const int last = min(t0 + p.tq, p.m) - 1;
    s_range[0] = upper_bound(p.kpos, p.Nc, p.qpos[last]);
    s_range[1] = upper_bound(p.kpos, p.Nc, p.qpos[t0]);
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const int kv_end = s_range[0];
  const int mask_from = s_range[1];
  const int n_tiles = (kv_end + BKV - 1) / BKV;

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      mbar_arrive_expect_tx(q_full, TILE_BYTES);
      tma_load_3d(sQ, &tmQ, q_full, 0, g * p.G, t0);
      tma_load_3d(sQ + CHUNK_BYTES, &tmQ, q_full, 64, g * p.G, t0);
      uint32_t issued = 0, issued_par = 0;
      for (int j = 0; j < n_tiles; ++j) {
        const int st = j % KV_STAGES;
        const uint32_t ph = (j / KV_STAGES) & 1;
        if (!mbar_wait(&kv_empty[st], ph ^ 1u, abort_flag, p.status, p.wait_ns, 0x21u)) break;
        mbar_arrive_expect_tx(&k_full[st], TILE_BYTES);
        tma_load_3d(sK + st * TILE_BYTES, &tmK, &k_full[st], 0, g, j * BKV);
        tma_load_3d(sK + st * TILE_BYTES + CHUNK_BYTES, &tmK, &k_full[st], 64, g, j * BKV);
        mbar_arrive_expect_tx(&v_full[st], TILE_BYTES);
        tma_load_3d(sV + st * TILE_BYTES, &tmV, &v_full[st], 0, g, j * BKV);
        tma_load_3d(sV + st * TILE_BYTES + CHUNK_BYTES, &tmV, &v_full[st], 64, g, j * BKV);
        issued |= 1u << st;
        issued_par = (issued_par & ~(1u << st)) | (ph << st);
      }
      if (*abort_flag) {
        mbar_drain(q_full, 0, p.status);
        for (int st = 0; st < KV_STAGES; ++st)
          if (issued & (1u << st)) {
            mbar_drain(&k_full[st], (issued_par >> st) & 1u, p.status);
            mbar_drain(&v_full[st], (issued_par >> st) & 1u, p.status);
          }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, BKV, 0, 0);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, 128, 0, 1);
      bool ok = mbar_wait(q_full, 0, abort_flag, p.status, p.wait_ns, 0x22u);
      tc_fence_after();
      const uint32_t q_addr = smem_u32(sQ);
      // S_j goes to TMEM buffer j % 2.  tcgen05.mma from this thread run in
      // issue order, so S_{j+2} (issued after PV_j) cannot overwrite P_j
      // before PV_j has read it.
      auto issue_s = [&](int j) -> bool {
        const int st = j % KV_STAGES;
        if (!mbar_wait(&k_full[st], (j / KV_STAGES) & 1, abort_flag, p.status, p.wait_ns, 0x23u)) return false;
        tc_fence_after();
        const uint32_t k_addr = smem_u32(sK + st * TILE_BYTES);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t a = sdesc_k_sw128(q_addr + (kk >> 2) * CHUNK_BYTES) + 2 * (kk & 3);
          const uint64_t b = sdesc_k_sw128(k_addr + (kk >> 2) * CHUNK_BYTES) + 2 * (kk & 3);
          mma_bf16_ss(tmem + (j & 1) * BKV, a, b, idesc_s, kk > 0);
        }
        tc_commit(&s_full[j & 1]);
        return true;
      };
      if (ok && n_tiles > 0) ok = issue_s(0);
      for (int j = 0; ok && j < n_tiles; ++j) {
        if (j + 1 < n_tiles && !issue_s(j + 1)) break;
        const int b = j & 1, st = j % KV_STAGES;
        if (!mbar_wait(&p_ready[b], (j >> 1) & 1, abort_flag, p.status, p.wait_ns, 0x24u)) break;
        if (!mbar_wait(&v_full[st], (j / KV_STAGES) & 1, abort_flag, p.status, p.wait_ns, 0x25u)) break;
        tc_fence_after();
        const uint32_t v_addr = smem_u32(sV + st * TILE_BYTES);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t v = sdesc_mn_sw128(v_addr + kk * 16 * 128, CHUNK_BYTES);
          mma_bf16_ts(tmem + 256, tmem + b * BKV + kk * 8, v, idesc_pv, (j | kk) != 0);
        }
        tc_commit(&kv_empty[st]);
        tc_commit(&p_free[b]);
      }
      tc_commit(drain);
      mbar_drain(drain, 0, p.status);
    }
    __syncwarp();
  } else {
    // softmax warps: TMEM lane quadrant = warp % 4
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const int tok = t0 + r / p.G;
    const bool valid = tok < p.m;
    const int32_t qp = valid ? p.qpos[tok] : INT_MIN;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    const float c2 = p.scale_log2;
    float m_run = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < n_tiles; ++j) {
      const int b = j & 1;
      ok = mbar_wait(&s_full[b], (j >> 1) & 1, abort_flag, p.status, p.wait_ns, 0x26u);
      if (!__all_sync(0xffffffffu, ok)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t xr[BKV];
#pragma unroll
      for (int c = 0; c < 4; ++c)
        tmem_ld32(lane_base + b * BKV + c * 32, *reinterpret_cast<uint32_t(*)[32]>(xr + 32 * c));
      tmem_ld_wait();
      // raw scores; the scale (> 0) is folded into the row max and the exp2 FFMA
      float x[BKV];
#pragma unroll
      for (int c = 0; c < BKV; ++c) x[c] = __uint_as_float(xr[c]);
      const int j0 = j * BKV;
      const bool need_mask = (j0 + BKV > mask_from) || (j0 + BKV > kv_end);
      if (need_mask) {
#pragma unroll
        for (int c = 0; c < BKV; ++c) {
          const int key = j0 + c;
          if (!(key < kv_end && __ldg(p.kpos + key) <= qp)) x[c] = -INFINITY;
        }
      }
      float m8[8];
#pragma unroll
      for (int t = 0; t < 8; ++t) m8[t] = x[t];
#pragma unroll
      for (int c = 8; c < BKV; ++c) m8[c & 7] = fmaxf(m8[c & 7], x[c]);
      const float mt = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                             fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7]))) * c2;
      const float m_new = fmaxf(m_run, mt);
      const bool need = m_new > m_run + RESCALE_THRESHOLD;
      if (__any_sync(0xffffffffu, need)) {
        const float factor = (m_run == -INFINITY) ? 0.f : ex2(m_run - m_new);
        if (j > 0) {
          const int pb = (j - 1) & 1;
          const bool okw = mbar_wait(&p_free[pb], ((j - 1) >> 1) & 1, abort_flag, p.status, p.wait_ns, 0x27u);
          if (!__all_sync(0xffffffffu, okw)) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            uint32_t o[32];
            tmem_ld32(lane_base + 256 + c * 32, o);
            tmem_ld_wait();
#pragma unroll
            for (int t = 0; t < 32; ++t) o[t] = __float_as_uint(__uint_as_float(o[t]) * factor);
            tmem_st32(lane_base + 256 + c * 32, o);
          }
          tmem_st_wait();
        }
        l *= factor;
        m_run = m_new;
      }
      const float neg_m = (m_run == -INFINITY) ? 0.f : -m_run;
      float s8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t pk[32];
#pragma unroll
        for (int t = 0; t < 32; ++t) {
          const float e0 = ex2(fmaf(x[h * 64 + 2 * t], c2, neg_m));
          const float e1 = ex2(fmaf(x[h * 64 + 2 * t + 1], c2, neg_m));
          s8[(2 * t) & 7] += e0;
          s8[(2 * t + 1) & 7] += e1;
          pk[t] = pack_bf16x2(e0, e1);
        }
        // P over the S values of this buffer: columns [b*128 + 32h, +32) hold keys [64h, 64h+64)
        tmem_st32(lane_base + b * BKV + h * 32, pk);
      }
      l += ((s8[0] + s8[1]) + (s8[2] + s8[3])) + ((s8[4] + s8[5]) + (s8[6] + s8[7]));
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&p_ready[b]);
    }
    // final normalisation once the last PV has landed
    if (ok && n_tiles > 0) {
      const int pb = (n_tiles - 1) & 1;
      const bool okw = mbar_wait(&p_free[pb], ((n_tiles - 1) >> 1) & 1, abort_flag, p.status, p.wait_ns, 0x29u);
      ok = __all_sync(0xffffffffu, okw);
      if (ok) tc_fence_after();
    }
    if (ok) {  // warp-uniform: the TMEM loads below are warp-collective
      const float inv = l > 0.f ? 1.f / l : 0.f;
      __nv_bfloat16 *orow = p.o + (static_cast<int64_t>(valid ? tok : 0) * p.Hq + g * p.G + r % p.G) * 128;
      if (n_tiles > 0) {
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t o[32];
          tmem_ld32(lane_base + 256 + c * 32, o);
          tmem_ld_wait();
          if (valid) {
            uint4 *dst = reinterpret_cast<uint4 *>(orow + c * 32);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              uint4 v;
              v.x = pack_bf16x2(__uint_as_float(o[8 * q + 0]) * inv, __uint_as_float(o[8 * q + 1]) * inv);
              v.y = pack_bf16x2(__uint_as_float(o[8 * q + 2]) * inv, __uint_as_float(o[8 * q + 3]) * inv);
              v.z = pack_bf16x2(__uint_as_float(o[8 * q + 4]) * inv, __uint_as_float(o[8 * q + 5]) * inv);
              v.w = pack_bf16x2(__uint_as_float(o[8 * q + 6]) * inv, __uint_as_float(o[8 * q + 7]) * inv);
              dst[q] = v;
            }
          }
        }
      } else if (valid) {
        uint4 *dst = reinterpret_cast<uint4 *>(orow);
        for (int q = 0; q < 16; ++q) dst[q] = make_uint4(0, 0, 0, 0);
      }
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace

spts_status launch_attention_bf16(const void *q, const int32_t *qpos, int64_t m, const void *k, const void *v,
                                  const int32_t *kpos, int64_t Nc, int Hq, int Hkv, float scale, void *o,
                                  uint32_t *status, cudaStream_t s) {
  if (m == 0) return SPTS_OK;
  const int G = Hq / Hkv;
  const int tq = 128 / G;
  CUtensorMap tq_map, tk_map, tv_map;
  {
    uint64_t dims[3] = {128, static_cast<uint64_t>(Hq), static_cast<uint64_t>(m)};
    uint64_t strides[2] = {128 * 2, static_cast<uint64_t>(Hq) * 128 * 2};
    uint32_t box[3] = {64, static_cast<uint32_t>(G), static_cast<uint32_t>(tq)};
    SPTS_TRY(make_tmap(&tq_map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, q, dims, strides, box,
                       CU_TENSOR_MAP_SWIZZLE_128B));
  }
  {
    uint64_t dims[3] = {128, static_cast<uint64_t>(Hkv), static_cast<uint64_t>(Nc)};
    uint64_t strides[2] = {128 * 2, static_cast<uint64_t>(Hkv) * 128 * 2};
    uint32_t box[3] = {64, 1, BKV};
    SPTS_TRY(make_tmap(&tk_map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, k, dims, strides, box,
                       CU_TENSOR_MAP_SWIZZLE_128B));
    SPTS_TRY(make_tmap(&tv_map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, v, dims, strides, box,
                       CU_TENSOR_MAP_SWIZZLE_128B));
  }
  Params p{};
  p.qpos = qpos;
  p.kpos = kpos;
  p.o = static_cast<__nv_bfloat16 *>(o);
  p.m = static_cast<int>(m);
  p.Nc = static_cast<int>(Nc);
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = G;
  p.tq = tq;
  p.n_qtiles = static_cast<int>((m + tq - 1) / tq);
  p.scale_log2 = scale * 1.4426950408889634f;
  p.status = status;
  p.wait_ns = wait_limit_ns();
  SPTS_CUDA_TRY(cudaFuncSetAttribute(attention_bf16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     static_cast<int>(SMEM_BYTES)));
  const unsigned grid = static_cast<unsigned>(p.n_qtiles) * static_cast<unsigned>(Hkv);
  attention_bf16_kernel<<<grid, THREADS, SMEM_BYTES, s>>>(tq_map, tk_map, tv_map, p);
  note_launch();
  SPTS_CUDA_TRY(cudaGetLastError());
  return SPTS_OK;
}

}  // namespace spts
