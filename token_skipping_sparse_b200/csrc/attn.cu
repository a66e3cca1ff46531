// attn.cu -- reduced GQA attention of SPTS on sm_100a (Fig. 2(a): the
// informative tokens attend to every candidate key, causally by original
// position).
//
// One CTA per (pair of Q tiles, KV head).  A Q tile packs 128/G selected
// tokens x the G query heads that share KV head g (G = Hq/Hkv); a CTA holds
// two consecutive Q tiles, A and B, so every K/V tile it loads feeds four
// M=128 MMAs (S and PV for each tile) and the softmax of one tile runs while
// the tensor core works on the other.
//   warp 0      TMA: both Q tiles and key tile 0 at entry (while warps 0..3
//               find the tiles' key ranges by warp-wide searches), then the
//               other K and V tiles of 128 keys into two 2-stage rings
//               (128-byte swizzle); a K stage is released once both tiles'
//               S MMAs have read it and a V stage once both PVs have, so the
//               next key tile's load does not wait for the PVs;
//   warp 1      MMA, per key tile j: PV_A(j), S_A(j+1), PV_B(j), S_B(j+1),
//               the whole warp running the loop on warp-uniform descriptors
//               and one elected lane issuing each tcgen05 op (a lone lane
//               under a lane test issued them markedly slower);
//               S_X = Q_X K^T lands in TMEM region S_X; the softmax writes
//               bf16 P over it and PV reads P from TMEM (A operand in TMEM)
//               with V an MN-major shared-memory operand, into O_X;
//   warps 2..3  idle (they complete warpgroup 0 for the register split);
//   warps 4..7  softmax of tile A, warps 8..11 softmax of tile B, one thread
//               per Q row: tcgen05.ld of the S row, causal mask (only on key
//               tiles crossing the tile's diagonal, against the row's last
//               visible key found once up front), row max with independent
//               three-input max accumulators, lazy O rescale (only when the
//               running max grows by more than 2^8), the scale folded into a
//               packed fp32x2 FFMA before exp2, row sums in packed fp32x2
//               adds, bf16 P back to TMEM; at the end O / l -> bf16.
// Tile A holds the earlier tokens, so its key range is a prefix of B's: the
// MMA and the softmax of A stop at A's own last visible key.  CTAs run in
// groups of HEAD_GROUP KV heads (the K/V they walk then fits in L2); inside a
// group pairs are launched latest-first so the long ones start early.  Part
// of each softmax row's exp2 runs on the FMA pipe (exp2_poly2).
// All barrier waits are bounded (see sm100.cuh).
#include <climits>

#include "host.hpp"
#include "rowops.cuh"
#include "sm100.cuh"

namespace spts {
namespace {

constexpr int THREADS = 384;
// setmaxnreg split: each SMSP holds one warp of warpgroup 0 and one softmax
// warp of each tile: 56 + 2 x 224 = 3 x 168, the launch allocation.
constexpr int REG_LOW = 56, REG_HIGH = 224;
constexpr int BKV = 128;
constexpr int KV_STAGES = 2;
constexpr int TILE_BYTES = 128 * 128 * 2;  // 32 KB: 128 rows x 128 bf16, as two 64-wide swizzled chunks
constexpr int CHUNK_BYTES = 128 * 64 * 2;  // 16 KB
constexpr int OFF_Q = 0;                                // Q_A, Q_B
constexpr int OFF_K = OFF_Q + 2 * TILE_BYTES;           // KV_STAGES stages
constexpr int OFF_V = OFF_K + KV_STAGES * TILE_BYTES;   // KV_STAGES stages
constexpr int OFF_BAR = OFF_V + KV_STAGES * TILE_BYTES;
constexpr size_t SMEM_BYTES = OFF_BAR + 256;
constexpr uint32_t TMEM_COLS = 512;  // S_A [0,128), S_B [128,256), O_A [256,384), O_B [384,512)
constexpr float RESCALE_THRESHOLD = 8.0f;  // log2 units
// One column pair in POLY_EVERY takes its exp2 from the polynomial on the
// FMA pipe (exp2_poly2), the others from the MUFU pipe, which alone would
// need as many cycles per key tile as the tile's two MMAs.
#ifndef SPTS_ATTN_POLY_EVERY
#define SPTS_ATTN_POLY_EVERY 3
#endif
constexpr int POLY_EVERY = SPTS_ATTN_POLY_EVERY;
// KV heads per scheduling group: CTAs run group by group (pairs latest-first
// inside a group), so the K/V that resident CTAs walk is the group's alone
// and stays in L2 instead of being fetched from HBM several times.  Two
// heads while their K/V (512 B per key and head) stays within ~48 MB, one
// head beyond (a model of the dispatch with LRU over 64 KB K/V tiles and
// ~60 MB of effective L2: 32K keys, two heads: 128 MB of K/V read, the
// floor; 128K keys: 0.77 GB with one head against 1.5 GB with two).
constexpr int HEAD_GROUP = 2;
constexpr int64_t HEAD_GROUP_MAX_KEYS = 49152;

struct Params {
  const int32_t *qpos;
  const int32_t *kpos;
  __nv_bfloat16 *o;
  int m, Nc, Hq, Hkv, G, tq, n_pairs, hgroup;
  float scale_log2;
  uint32_t *status;
  uint64_t wait_ns;
};

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// A three-input max: with the packed f32x2 arithmetic of sm100.cuh it
// halves the instruction count of the softmax's per-element work.
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

__global__ void __launch_bounds__(THREADS, 1)
    attention_bf16_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                          const __grid_constant__ CUtensorMap tmV, const __grid_constant__ Params p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t *sQ = smem + OFF_Q;
  uint8_t *sK = smem + OFF_K;
  uint8_t *sV = smem + OFF_V;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
  uint64_t *q_full = bars + 0, *k_full = bars + 1, *v_full = k_full + KV_STAGES, *k_empty = v_full + KV_STAGES,
           *v_empty = k_empty + KV_STAGES, *s_full = v_empty + KV_STAGES, *p_ready = s_full + 2,
           *o_done = p_ready + 4, *drain = o_done + 2;
  // p_ready[2 X + h]: P of tile X for keys [64 h, 64 h + 64) is in TMEM
  uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(drain + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);
  int *s_range = reinterpret_cast<int *>(tmem_holder + 2);  // per tile X: kv_end[X], mask_from[X]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int per_group = p.n_pairs * p.hgroup;
  const int rem = static_cast<int>(blockIdx.x) % per_group;
  const int pair = p.n_pairs - 1 - rem / p.hgroup;
  const int g = static_cast<int>(blockIdx.x) / per_group * p.hgroup + rem % p.hgroup;
  const int t0 = pair * 2 * p.tq;  // first token of tile A; tile B starts at t0 + tq

  if (smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0) raise_status(p.status, SPTS_DEV_BADINDEX, 0x2Fu, smem_u32(smem));
    return;
  }
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < KV_STAGES; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&s_full[x], 1);
      mbar_init(&p_ready[2 * x], 128);
      mbar_init(&p_ready[2 * x + 1], 128);
      mbar_init(&o_done[x], 1);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    // both Q tiles and key tile 0 (where every tile's key loop starts) are
    // in flight while the key ranges are searched
    mbar_arrive_expect_tx(q_full, 2 * TILE_BYTES);
    for (int x = 0; x < 2; ++x) {
      tma_load_3d(sQ + x * TILE_BYTES, &tmQ, q_full, 0, g * p.G, t0 + x * p.tq);
      tma_load_3d(sQ + x * TILE_BYTES + CHUNK_BYTES, &tmQ, q_full, 64, g * p.G, t0 + x * p.tq);
    }
    mbar_arrive_expect_tx(&k_full[0], TILE_BYTES);
    tma_load_3d(sK, &tmK, &k_full[0], 0, g, 0);
    tma_load_3d(sK + CHUNK_BYTES, &tmK, &k_full[0], 64, g, 0);
    mbar_arrive_expect_tx(&v_full[0], TILE_BYTES);
    tma_load_3d(sV, &tmV, &v_full[0], 0, g, 0);
    tma_load_3d(sV + CHUNK_BYTES, &tmV, &v_full[0], 64, g, 0);
  }
  // Key ranges of the two tiles, one warp-wide search each on warps 0..3:
  // kv_end[X] = keys at or before the tile's last query, mask_from[X] = keys
  // at or before its first (a tile beyond the last token has no work).
  if (warp < 4) {
    const int x = warp >> 1, first = t0 + x * p.tq;
    int r = 0;
    if (first < p.m) r = warp_upper_bound(p.kpos, p.Nc, p.qpos[(warp & 1) ? first : min(first + p.tq, p.m) - 1]);
    if (lane == 0) s_range[2 * x + (warp & 1)] = r;
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const int n_a = (s_range[0] + BKV - 1) / BKV;
  const int n_b = (s_range[2] + BKV - 1) / BKV;
  const int n_kv = max(n_a, n_b);

  if (warp == 0) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(REG_LOW));
    if (lane == 0) {
      // K and V stages are released separately (K tile j once both tiles'
      // S(j) have completed, V tile j once both PV(j) have)
      uint32_t k_issued = 1u, k_par = 0, v_issued = 1u, v_par = 0;  // stage 0: key tile 0, loaded at entry
      for (int j = 1; j < n_kv; ++j) {
        const int st = j % KV_STAGES;
        const uint32_t ph = (j / KV_STAGES) & 1;
        if (!mbar_wait(&k_empty[st], ph ^ 1u, abort_flag, p.status, p.wait_ns, 0x21u)) break;
        mbar_arrive_expect_tx(&k_full[st], TILE_BYTES);
        tma_load_3d(sK + st * TILE_BYTES, &tmK, &k_full[st], 0, g, j * BKV);
        tma_load_3d(sK + st * TILE_BYTES + CHUNK_BYTES, &tmK, &k_full[st], 64, g, j * BKV);
        k_issued |= 1u << st;
        k_par = (k_par & ~(1u << st)) | (ph << st);
        if (!mbar_wait(&v_empty[st], ph ^ 1u, abort_flag, p.status, p.wait_ns, 0x2Au)) break;
        mbar_arrive_expect_tx(&v_full[st], TILE_BYTES);
        tma_load_3d(sV + st * TILE_BYTES, &tmV, &v_full[st], 0, g, j * BKV);
        tma_load_3d(sV + st * TILE_BYTES + CHUNK_BYTES, &tmV, &v_full[st], 64, g, j * BKV);
        v_issued |= 1u << st;
        v_par = (v_par & ~(1u << st)) | (ph << st);
      }
      if (n_kv == 0) {  // no visible key: let the entry loads of tile 0 land
        mbar_drain(&k_full[0], 0, p.status);
        mbar_drain(&v_full[0], 0, p.status);
      }
      if (*abort_flag) {
        mbar_drain(q_full, 0, p.status);
        for (int st = 0; st < KV_STAGES; ++st) {
          if (k_issued & (1u << st)) mbar_drain(&k_full[st], (k_par >> st) & 1u, p.status);
          if (v_issued & (1u << st)) mbar_drain(&v_full[st], (v_par >> st) & 1u, p.status);
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(REG_LOW));
    {  // the whole warp runs the issue loop; one elected lane issues each MMA and commit
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, BKV, 0, 0);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, 128, 0, 1);
      auto wait_all = [&](uint64_t *bar, uint32_t parity, uint32_t where) -> bool {
        return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, p.status, p.wait_ns, where));
      };
      bool ok = wait_all(q_full, 0, 0x22u);
      tc_fence_after();
      // S_X(j) into TMEM region S_X.  tcgen05.mma from this thread run in
      // issue order, so S_X(j+1) (issued after PV_X(j)) cannot overwrite P_X(j)
      // before PV_X(j) has read it.
      auto issue_s = [&](int x, int j) -> bool {
        const int st = j % KV_STAGES;
        if (!wait_all(&k_full[st], (j / KV_STAGES) & 1, 0x23u)) return false;
        tc_fence_after();
        const uint32_t k_addr = smem_u32(sK + st * TILE_BYTES);
        const uint32_t q_addr = smem_u32(sQ + x * TILE_BYTES);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t a = sdesc_k_sw128(q_addr + (kk >> 2) * CHUNK_BYTES) + 2 * (kk & 3);
          const uint64_t b = sdesc_k_sw128(k_addr + (kk >> 2) * CHUNK_BYTES) + 2 * (kk & 3);
          mma_bf16_ss_w(tmem + x * BKV, a, b, idesc_s, kk > 0);
        }
        tc_commit_w(&s_full[x]);
        return true;
      };
      // PV in two halves of 64 keys, each issued as soon as the softmax has
      // stored that half of P: the first half runs while the softmax is
      // still on the second.
      auto issue_pv = [&](int x, int j) -> bool {
        const int st = j % KV_STAGES;
        if (!wait_all(&v_full[st], (j / KV_STAGES) & 1, 0x25u)) return false;
        const uint32_t v_addr = smem_u32(sV + st * TILE_BYTES);
        for (int half = 0; half < 2; ++half) {
          if (!wait_all(&p_ready[2 * x + half], j & 1, 0x24u)) return false;
          tc_fence_after();
#pragma unroll
          for (int kq = 0; kq < 4; ++kq) {
            const int kk = 4 * half + kq;
            const uint64_t v = sdesc_mn_sw128(v_addr + kk * 16 * 128, CHUNK_BYTES);
            mma_bf16_ts_w(tmem + 256 + x * 128, tmem + x * BKV + kk * 8, v, idesc_pv, (j | kk) != 0);
          }
        }
        tc_commit_w(&o_done[x]);
        return true;
      };
      for (int x = 0; ok && x < 2; ++x)
        if ((x == 0 ? n_a : n_b) > 0) ok = issue_s(x, 0);
      if (ok && n_kv > 0) tc_commit_w(&k_empty[0]);  // both S(0) read key tile 0
      for (int j = 0; ok && j < n_kv; ++j) {
        for (int x = 0; ok && x < 2; ++x) {
          const int nxx = x == 0 ? n_a : n_b;
          if (j >= nxx) continue;
          ok = issue_pv(x, j);
          if (ok && j + 1 < nxx) ok = issue_s(x, j + 1);
        }
        if (!ok) break;
        // V tile j is free once both PV(j) are done, key tile j + 1 once both
        // S(j+1) are: the next key tile's load no longer waits for the PVs
        tc_commit_w(&v_empty[j % KV_STAGES]);
        if (j + 1 < n_kv) tc_commit_w(&k_empty[(j + 1) % KV_STAGES]);
      }
      tc_commit_w(drain);
      mbar_drain(drain, 0, p.status);
    }
    __syncwarp();
  } else if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(REG_LOW));  // idle
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(REG_HIGH));
    // ---------------- softmax: warps 4..7 tile A, warps 8..11 tile B
    const int x = (warp - 4) >> 2;
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const int tok = t0 + x * p.tq + r / p.G;
    const bool valid = tok < p.m;
    const int32_t qp = valid ? p.qpos[tok] : INT_MIN;
    const int kv_end = s_range[2 * x], mask_from = s_range[2 * x + 1];
    // This row sees keys [0, lim): kpos ascending, so lim = keys at or before
    // its query, between the tile's mask_from and kv_end (0 for padding rows).
    // Found once here, while the first S tile is on its way.
    int lim = 0;
    if (valid) {
      int lo = mask_from, hi = kv_end;
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (__ldg(p.kpos + mid) <= qp) lo = mid + 1;
        else hi = mid;
      }
      lim = lo;
    }
    const int n_tiles = x == 0 ? n_a : n_b;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    const uint32_t s_col = x * BKV, o_col = 256 + x * 128;
    const float c2 = p.scale_log2;
    float m_run = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < n_tiles; ++j) {
      ok = mbar_wait(&s_full[x], j & 1, abort_flag, p.status, p.wait_ns, 0x26u);
      if (!__all_sync(0xffffffffu, ok)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t xr[BKV];
#pragma unroll
      for (int c = 0; c < 4; ++c)
        tmem_ld32(lane_base + s_col + c * 32, *reinterpret_cast<uint32_t(*)[32]>(xr + 32 * c));
      tmem_ld_wait();
      const int j0 = j * BKV;
      // causal mask, only on key tiles past the tile's first query (which
      // includes every tile reaching past kv_end >= mask_from)
      if (j0 + BKV > mask_from) {
        const int vis = lim - j0;
#pragma unroll
        for (int c = 0; c < BKV; ++c)
          if (c >= vis) xr[c] = 0xff800000u;  // -inf
      }
      float m8[8];
#pragma unroll
      for (int t = 0; t < 8; ++t) m8[t] = __uint_as_float(xr[t]);
#pragma unroll
      for (int c = 8; c < BKV; c += 2)
        m8[(c >> 1) & 7] = fmax3(m8[(c >> 1) & 7], __uint_as_float(xr[c]), __uint_as_float(xr[c + 1]));
      const float mt = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                             fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7]))) * c2;
      const float m_new = fmaxf(m_run, mt);
      const bool need = m_new > m_run + RESCALE_THRESHOLD;
      if (__any_sync(0xffffffffu, need)) {
        const float factor = (m_run == -INFINITY) ? 0.f : ex2(m_run - m_new);
        if (j > 0) {  // O_X holds PV_X(0..j-1): wait for the last of them
          const bool okw = mbar_wait(&o_done[x], (j - 1) & 1, abort_flag, p.status, p.wait_ns, 0x27u);
          if (!__all_sync(0xffffffffu, okw)) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            uint32_t o[32];
            tmem_ld32(lane_base + o_col + c * 32, o);
            tmem_ld_wait();
#pragma unroll
            for (int t = 0; t < 32; ++t) o[t] = __float_as_uint(__uint_as_float(o[t]) * factor);
            tmem_st32(lane_base + o_col + c * 32, o);
          }
          tmem_st_wait();
        }
        l *= factor;
        m_run = m_new;
      }
      const float neg_m = (m_run == -INFINITY) ? 0.f : -m_run;
      const uint64_t cc = f2pack(c2, c2), mm = f2pack(neg_m, neg_m);
      uint64_t s4[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t pk[32];
#pragma unroll
        for (int t = 0; t < 32; ++t) {
          const uint64_t a2 =
              f2fma(f2pack(__uint_as_float(xr[h * 64 + 2 * t]), __uint_as_float(xr[h * 64 + 2 * t + 1])), cc, mm);
          float e0, e1;
          if (t % POLY_EVERY == POLY_EVERY - 1) {  // this pair on the FMA pipe
            exp2_poly2(a2, e0, e1);
          } else {
            float a0, a1;
            f2unpack(a2, a0, a1);
            e0 = ex2(a0);
            e1 = ex2(a1);
          }
          s4[t & 3] = f2add(s4[t & 3], f2pack(e0, e1));
          pk[t] = pack_bf16x2(e0, e1);
        }
        // P over this tile's S values: columns [32h, 32h+32) hold keys [64h, 64h+64)
        tmem_st32(lane_base + s_col + h * 32, pk);
        if (h == 0) {  // the first half of P is in place: its PV can start
          tmem_st_wait();
          tc_fence_before();
          mbar_arrive(&p_ready[2 * x]);
        }
      }
      {
        float q0, q1, q2, q3, q4, q5, q6, q7;
        f2unpack(f2add(s4[0], s4[1]), q0, q1);
        f2unpack(f2add(s4[2], s4[3]), q2, q3);
        (void)q4; (void)q5; (void)q6; (void)q7;
        l += (q0 + q1) + (q2 + q3);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&p_ready[2 * x + 1]);
    }
    // final normalisation once the last PV of this tile has landed
    if (ok && n_tiles > 0) {
      const bool okw = mbar_wait(&o_done[x], (n_tiles - 1) & 1, abort_flag, p.status, p.wait_ns, 0x29u);
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
          tmem_ld32(lane_base + o_col + c * 32, o);
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
  p.n_pairs = static_cast<int>((m + 2 * tq - 1) / (2 * tq));
  p.hgroup = (Hkv % HEAD_GROUP == 0 && Nc <= HEAD_GROUP_MAX_KEYS) ? HEAD_GROUP : 1;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.status = status;
  p.wait_ns = wait_limit_ns();
  SPTS_CUDA_TRY(cudaFuncSetAttribute(attention_bf16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     static_cast<int>(SMEM_BYTES)));
  const unsigned grid = static_cast<unsigned>(p.n_pairs) * static_cast<unsigned>(Hkv);
  attention_bf16_kernel<<<grid, THREADS, SMEM_BYTES, s>>>(tq_map, tk_map, tv_map, p);
  note_launch();
  SPTS_CUDA_TRY(cudaGetLastError());
  return SPTS_OK;
}

}  // namespace spts
