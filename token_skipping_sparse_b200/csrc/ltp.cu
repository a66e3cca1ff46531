// ltp.cu -- Low-rank Transformation Probing score on sm_100a (Fig. 2(b),
// Table 6, Table A): c_i = || (x_i A^T) B^T ||_2.
//
// One CTA per tile of 128 rows, a chained pair of tcgen05 GEMMs that never
// writes the proxy output to memory:
//   phase 1  T = X A^T   (M=128, N=r, K=D) accumulated in TMEM, then read
//            back, rounded to bf16 and stored in shared memory in the UMMA
//            K-major swizzled layout, where it becomes the A operand of
//   phase 2  for the L2 norm, U = T G with the Gram matrix G = B^T B (r x r,
//            built per call, as two bf16 halves G_hi + G_lo): ||T B^T||^2 =
//            rowsum(T * U), so phase 2 costs r x r instead of r x Dout per
//            row (Dout = 4096, r = 256: 16x less); T stays in TMEM beside U.
// With top_m > 0 (D_low = Dout <= 512) phase 2 is Y = T B^T (M=128, N=256 per
// chunk, K=r), both chunks resident in TMEM, and the
// score is instead the sum of the top_m largest |y| of the row (top-rho
// channel saliency, Table E): each row's thread searches the float bits of
// |y| from the top for a threshold with exactly top_m values at or above it
// (counting passes over the row in TMEM, at most 31, usually about half),
// then sums the values above it plus the ties at it that top_m needs.
// Per row only 2*D bytes of X are read from HBM; A, B and G are shared by
// all CTAs through L2.  Waits are bounded.
#include "host.hpp"
#include "rowops.cuh"
#include "sm100.cuh"

namespace spts {
namespace {

constexpr int THREADS = 192;
constexpr int STAGES = 3;
constexpr int SLOT = 48 * 1024;
constexpr int X_BYTES = 128 * 64 * 2;  // 16 KB
constexpr int CHUNK_BYTES = 128 * 64 * 2;
constexpr int OFF_TS = STAGES * SLOT;               // T in bf16: r/64 chunks of 16 KB
constexpr int OFF_BAR = OFF_TS + 4 * CHUNK_BYTES;
constexpr size_t SMEM_BYTES = 1024 + OFF_BAR + 256;

struct Params {
  int M, D, r, Dout;
  int top_m;  // 0: L2 norm of y through the Gram form; > 0: sum of the top_m largest |y| (Dout <= 512)
  float *scores;
  uint32_t *status;
  uint64_t wait_ns;
};

__global__ void __launch_bounds__(THREADS, 1)
    ltp_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmA,
               const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmGhi,
               const __grid_constant__ CUtensorMap tmGlo, const __grid_constant__ Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sT = smem + OFF_TS;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
  uint64_t *full = bars, *empty = bars + STAGES, *t_full = bars + 2 * STAGES, *ts_ready = t_full + 1,
           *acc_full = ts_ready + 1, *acc_empty = acc_full + 2, *drain = acc_empty + 2;
  uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(drain + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * 128;
  const int kb1 = p.D / 64, kb2 = p.r / 64, nch = p.Dout / 256;
  const bool gram = p.top_m == 0;  // phase 2 against G_hi, then G_lo (r x r each)

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(t_full, 1);
    mbar_init(ts_ready, 128);
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 128);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tmX);
      tma_prefetch_desc(&tmA);
      if (gram) {
        tma_prefetch_desc(&tmGhi);
        tma_prefetch_desc(&tmGlo);
      } else {
        tma_prefetch_desc(&tmB);
      }
      uint32_t issued = 0, par = 0;
      const int total = kb1 + (gram ? 2 * kb2 : nch * kb2);
      for (int i = 0; i < total; ++i) {
        const int st = i % STAGES;
        const uint32_t ph = (i / STAGES) & 1;
        if (!mbar_wait(&empty[st], ph ^ 1u, abort_flag, p.status, p.wait_ns, 0x51u)) break;
        uint8_t *slot = smem + st * SLOT;
        if (i < kb1) {
          mbar_arrive_expect_tx(&full[st], X_BYTES + p.r * 128);
          tma_load_2d(slot, &tmX, &full[st], i * 64, m0);
          tma_load_2d(slot + X_BYTES, &tmA, &full[st], i * 64, 0);
        } else if (gram) {  // G_hi k-blocks, then G_lo k-blocks: r rows x 64 columns
          const int j = i - kb1;
          mbar_arrive_expect_tx(&full[st], p.r * 128);
          tma_load_2d(slot, j < kb2 ? &tmGhi : &tmGlo, &full[st], (j % kb2) * 64, 0);
        } else {
          const int j = i - kb1;
          mbar_arrive_expect_tx(&full[st], 256 * 128);
          tma_load_2d(slot, &tmB, &full[st], (j % kb2) * 64, (j / kb2) * 256);
        }
        issued |= 1u << st;
        par = (par & ~(1u << st)) | (ph << st);
      }
      if (*abort_flag)
        for (int st = 0; st < STAGES; ++st)
          if (issued & (1u << st)) mbar_drain(&full[st], (par >> st) & 1u, p.status);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc1 = idesc_bf16_f32(128, p.r, 0, 0);
      constexpr uint32_t idesc2 = idesc_bf16_f32(128, 256, 0, 0);
      bool ok = true;
      int i = 0;
      for (int kb = 0; ok && kb < kb1; ++kb, ++i) {
        const int st = i % STAGES;
        if (!mbar_wait(&full[st], (i / STAGES) & 1, abort_flag, p.status, p.wait_ns, 0x52u)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t base = smem_u32(smem + st * SLOT);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16_ss(tmem, sdesc_k_sw128(base) + 2 * kk, sdesc_k_sw128(base + X_BYTES) + 2 * kk, idesc1,
                      (kb | kk) != 0);
        tc_commit(&empty[st]);
      }
      if (ok) tc_commit(t_full);
      if (ok) ok = mbar_wait(ts_ready, 0, abort_flag, p.status, p.wait_ns, 0x53u);
      tc_fence_after();
      const uint32_t t_addr = smem_u32(sT);
      if (gram && ok) {  // U = T G_hi^T + T G_lo^T into TMEM columns [256, 256 + r); T stays at [0, r)
        const uint32_t idesc_g = idesc_bf16_f32(128, p.r, 0, 0);
        for (int j = 0; ok && j < 2 * kb2; ++j, ++i) {
          const int st = i % STAGES;
          if (!mbar_wait(&full[st], (i / STAGES) & 1, abort_flag, p.status, p.wait_ns, 0x59u)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const int kb = j % kb2;
          const uint32_t base = smem_u32(smem + st * SLOT);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16_ss(tmem + 256, sdesc_k_sw128(t_addr + kb * CHUNK_BYTES) + 2 * kk, sdesc_k_sw128(base) + 2 * kk,
                        idesc_g, (j | kk) != 0);
          tc_commit(&empty[st]);
        }
        if (ok) tc_commit(&acc_full[0]);
      }
      for (int nc = 0; ok && !gram && nc < nch; ++nc) {
        const int acc = nc & 1;
        if (!mbar_wait(&acc_empty[acc], ((nc >> 1) & 1) ^ 1u, abort_flag, p.status, p.wait_ns, 0x54u)) break;
        tc_fence_after();
        for (int kb = 0; kb < kb2; ++kb, ++i) {
          const int st = i % STAGES;
          if (!mbar_wait(&full[st], (i / STAGES) & 1, abort_flag, p.status, p.wait_ns, 0x55u)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t base = smem_u32(smem + st * SLOT);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16_ss(tmem + acc * 256, sdesc_k_sw128(t_addr + kb * CHUNK_BYTES) + 2 * kk,
                        sdesc_k_sw128(base) + 2 * kk, idesc2, (kb | kk) != 0);
          tc_commit(&empty[st]);
        }
        if (ok) tc_commit(&acc_full[acc]);
      }
      tc_commit(drain);
      mbar_drain(drain, 0, p.status);
    }
    __syncwarp();
  } else {
    const int quad = warp & 3;
    const int rr = quad * 32 + lane;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    bool ok = mbar_wait(t_full, 0, abort_flag, p.status, p.wait_ns, 0x56u);
    ok = __all_sync(0xffffffffu, ok);
    if (ok) {
      tc_fence_after();
      // T row -> bf16 -> shared memory (K-major, 128-byte swizzle)
      for (int c0 = 0; c0 < p.r; c0 += 32) {
        uint32_t t[32];
        tmem_ld32(lane_base + c0, t);
        tmem_ld_wait();
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint4 v;
          v.x = pack_bf16x2(__uint_as_float(t[8 * q + 0]), __uint_as_float(t[8 * q + 1]));
          v.y = pack_bf16x2(__uint_as_float(t[8 * q + 2]), __uint_as_float(t[8 * q + 3]));
          v.z = pack_bf16x2(__uint_as_float(t[8 * q + 4]), __uint_as_float(t[8 * q + 5]));
          v.w = pack_bf16x2(__uint_as_float(t[8 * q + 6]), __uint_as_float(t[8 * q + 7]));
          const int col = c0 + 8 * q;
          *reinterpret_cast<uint4 *>(sT + (col / 64) * CHUNK_BYTES + sw128_offset(rr, (col % 64) / 8)) = v;
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(ts_ready);
    }
    float ss = 0.f;
    if (p.top_m > 0) {
      // both chunks (Dout <= 512 columns) resident: acc 0 = columns [0, 256)
      for (int nc = 0; ok && nc < nch; ++nc) {
        const bool okw = mbar_wait(&acc_full[nc], 0, abort_flag, p.status, p.wait_ns, 0x58u);
        ok = __all_sync(0xffffffffu, okw);
      }
      if (ok) {
        tc_fence_after();
        // a T with exactly top_m values of |y| >= T, or else the top_m-th
        // largest |y| itself: bit by bit from the top (|y| bits order as
        // uints), stopping once exactly top_m values lie at or above T
        uint32_t T = 0u;
        int at_or_above = p.Dout;  // values >= T
#pragma unroll 1
        for (int b = 30; b >= 0 && __any_sync(0xffffffffu, at_or_above != p.top_m); --b) {
          const uint32_t cand = T | (1u << b);
          int cnt = 0;
#pragma unroll 1
          for (int c0 = 0; c0 < p.Dout; c0 += 32) {
            uint32_t y[32];
            tmem_ld32(lane_base + c0, y);  // warp-wide: every lane loads, finished ones included
            tmem_ld_wait();
#pragma unroll
            for (int t = 0; t < 32; ++t) cnt += (y[t] & 0x7FFFFFFFu) >= cand;
          }
          if (at_or_above != p.top_m && cnt >= p.top_m) {
            T = cand;
            at_or_above = cnt;
          }
        }
        int gt = 0;
#pragma unroll 1
        for (int c0 = 0; c0 < p.Dout; c0 += 32) {
          uint32_t y[32];
          tmem_ld32(lane_base + c0, y);
          tmem_ld_wait();
#pragma unroll
          for (int t = 0; t < 32; ++t) {
            const uint32_t u = y[t] & 0x7FFFFFFFu;
            if (u > T) {
              ss += __uint_as_float(u);
              ++gt;
            }
          }
        }
        ss += static_cast<float>(p.top_m - gt) * __uint_as_float(T);  // the ties at the threshold
        tc_fence_before();
        for (int nc = 0; nc < nch; ++nc) mbar_arrive(&acc_empty[nc]);
      }
      if (ok && m0 + rr < p.M) p.scores[m0 + rr] = ss;
    }
    if (gram) {  // c^2 = sum_j bf16(T_j) U_j with U = bf16(T) G: T at [0, r), U at [256, 256 + r)
      const bool okw = mbar_wait(&acc_full[0], 0, abort_flag, p.status, p.wait_ns, 0x5Au);
      ok = ok && __all_sync(0xffffffffu, okw);
      if (ok) {
        tc_fence_after();
#pragma unroll 1
        for (int c0 = 0; c0 < p.r; c0 += 32) {
          uint32_t t[32], u[32];
          tmem_ld32(lane_base + c0, t);
          tmem_ld32(lane_base + 256 + c0, u);
          tmem_ld_wait();
#pragma unroll
          for (int q = 0; q < 32; ++q)
            ss = fmaf(__bfloat162float(__float2bfloat16_rn(__uint_as_float(t[q]))), __uint_as_float(u[q]), ss);
        }
        if (m0 + rr < p.M) p.scores[m0 + rr] = sqrtf(fmaxf(ss, 0.f));
      }
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------- Gram form
// For the L2-norm score ||t B^T||^2 = t (B^T B) t^T, so the second product
// needs only the r x r Gram matrix G = B^T B instead of all Dout outputs.
// G is built per call from B: fp32 partial sums of the upper-triangle 64 x 64
// blocks over up to 32 slices of the Dout rows (products of two bf16 are
// exact in fp32), then summed in a fixed slice order -- deterministic, and
// symmetric by construction (the lower blocks are the upper ones mirrored)
// -- and split into bf16 G_hi = bf16(G), G_lo = bf16(G - G_hi) for the
// tensor core (G_hi + G_lo carries 16 significant bits).
constexpr int GRAM_MAX_SPLITS = 32;
constexpr int GRAM_ROWS = 32;  // B rows staged per step

__host__ __device__ inline int gram_splits(int Dout) {  // slices of a multiple of GRAM_ROWS rows each
  const int s = Dout / GRAM_ROWS;
  return s < GRAM_MAX_SPLITS ? s : GRAM_MAX_SPLITS;
}

// Block (jb, kb), jb <= kb (G is symmetric), of 64 x 64 entries of G over the
// rows of slice blockIdx.y; blockIdx.x enumerates the upper-triangle blocks.
// 256 threads, 4 x 4 entries each; B rows staged in shared memory as fp32.
__global__ void __launch_bounds__(256) gram_partial_kernel(const __nv_bfloat16 *__restrict__ B, int Dout, int r,
                                                           int splits, float *__restrict__ part) {
  __shared__ __align__(16) float sj[GRAM_ROWS][64];
  __shared__ __align__(16) float sk[GRAM_ROWS][64];
  const int nb = r / 64;
  int jb = 0, t = blockIdx.x;
  while (t >= nb - jb) {
    t -= nb - jb;
    ++jb;
  }
  const int kb = jb + t;
  const int j0 = jb * 64, k0 = kb * 64;
  const int rows = Dout / splits, o0 = blockIdx.y * rows;
  const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;
  const int lo = threadIdx.x >> 3, lc = (threadIdx.x & 7) * 8;  // staging: row, first of 8 columns
  float acc[4][4] = {};
  for (int ob = 0; ob < rows; ob += GRAM_ROWS) {
    const int64_t row = static_cast<int64_t>(o0 + ob + lo) * r;
    const uint4 vj = *reinterpret_cast<const uint4 *>(B + row + j0 + lc);
    const uint4 vk = *reinterpret_cast<const uint4 *>(B + row + k0 + lc);
    const uint32_t wj[4] = {vj.x, vj.y, vj.z, vj.w}, wk[4] = {vk.x, vk.y, vk.z, vk.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {  // bf16 -> fp32 is a 16-bit shift
      sj[lo][lc + 2 * q] = __uint_as_float(wj[q] << 16);
      sj[lo][lc + 2 * q + 1] = __uint_as_float(wj[q] & 0xFFFF0000u);
      sk[lo][lc + 2 * q] = __uint_as_float(wk[q] << 16);
      sk[lo][lc + 2 * q + 1] = __uint_as_float(wk[q] & 0xFFFF0000u);
    }
    __syncthreads();
#pragma unroll 8
    for (int o = 0; o < GRAM_ROWS; ++o) {
      const float4 a4 = *reinterpret_cast<const float4 *>(&sj[o][ty * 4]);
      const float4 b4 = *reinterpret_cast<const float4 *>(&sk[o][tx * 4]);
      const float a[4] = {a4.x, a4.y, a4.z, a4.w}, b[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int w = 0; w < 4; ++w) acc[q][w] = fmaf(a[q], b[w], acc[q][w]);
    }
    __syncthreads();
  }
  float *dst = part + static_cast<int64_t>(blockIdx.y) * r * r;
#pragma unroll
  for (int q = 0; q < 4; ++q)
    *reinterpret_cast<float4 *>(dst + (j0 + ty * 4 + q) * r + k0 + tx * 4) =
        make_float4(acc[q][0], acc[q][1], acc[q][2], acc[q][3]);
}

// G[j][k] = sum of the slices in order (entries below the diagonal blocks
// read their mirror), then G_hi = bf16(G), G_lo = bf16(G - G_hi).
__global__ void gram_finish_kernel(const float *__restrict__ part, int r, int splits, __nv_bfloat16 *__restrict__ g_hi,
                                   __nv_bfloat16 *__restrict__ g_lo) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= r * r) return;
  int j = i / r, k = i % r;
  if (j / 64 > k / 64) {
    const int t = j;
    j = k;
    k = t;
  }
  float g = 0.f;
  for (int s = 0; s < splits; ++s) g += part[static_cast<int64_t>(s) * r * r + j * r + k];
  const __nv_bfloat16 hi = __float2bfloat16_rn(g);
  g_hi[i] = hi;
  g_lo[i] = __float2bfloat16_rn(g - __bfloat162float(hi));
}

}  // namespace

size_t ltp_gram_bytes(int r) {
  const size_t rr = static_cast<size_t>(r > 0 ? r : 1) * (r > 0 ? r : 1);
  auto up = [](size_t n) { return (n + 255) / 256 * 256; };
  return 2 * up(rr * 2) + up(static_cast<size_t>(GRAM_MAX_SPLITS) * rr * 4);
}

spts_status launch_ltp_bf16(const void *x, int64_t Nc, int D, const void *A, int r, const void *B, int Dout,
                            float *scores, uint32_t *status, cudaStream_t s, int top_m, void *gram_ws) {
  if (Nc == 0) return SPTS_OK;
  CUtensorMap tx, ta, tb, tghi, tglo;
  SPTS_TRY(tmap_bf16_2d(&tx, x, static_cast<uint64_t>(Nc), D, D, 128));
  SPTS_TRY(tmap_bf16_2d(&ta, A, r, D, D, static_cast<uint32_t>(r)));
  SPTS_TRY(tmap_bf16_2d(&tb, B, Dout, r, r, 256));
  if (top_m == 0) {  // the Gram form: G = B^T B, then its bf16 halves
    SPTS_REQUIRE(gram_ws != nullptr, SPTS_ERR_WORKSPACE, "ltp: no scratch for the Gram matrix");
    const size_t rr = static_cast<size_t>(r) * r;
    auto up = [](size_t n) { return (n + 255) / 256 * 256; };
    uint8_t *w = static_cast<uint8_t *>(gram_ws);
    __nv_bfloat16 *g_hi = reinterpret_cast<__nv_bfloat16 *>(w);
    __nv_bfloat16 *g_lo = reinterpret_cast<__nv_bfloat16 *>(w + up(rr * 2));
    float *part = reinterpret_cast<float *>(w + 2 * up(rr * 2));
    const int nb = r / 64, splits = gram_splits(Dout);
    gram_partial_kernel<<<dim3(nb * (nb + 1) / 2, splits), 256, 0, s>>>(static_cast<const __nv_bfloat16 *>(B), Dout,
                                                                        r, splits, part);
    note_launch();
    gram_finish_kernel<<<static_cast<unsigned>((rr + 255) / 256), 256, 0, s>>>(part, r, splits, g_hi, g_lo);
    note_launch();
    SPTS_TRY(tmap_bf16_2d(&tghi, g_hi, r, r, r, static_cast<uint32_t>(r)));
    SPTS_TRY(tmap_bf16_2d(&tglo, g_lo, r, r, r, static_cast<uint32_t>(r)));
  } else {
    tghi = tb;
    tglo = tb;
  }
  Params p{static_cast<int>(Nc), D, r, Dout, top_m, scores, status, wait_limit_ns()};
  SPTS_CUDA_TRY(
      cudaFuncSetAttribute(ltp_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(SMEM_BYTES)));
  ltp_kernel<<<static_cast<unsigned>((Nc + 127) / 128), THREADS, SMEM_BYTES, s>>>(tx, ta, tb, tghi, tglo, p);
  note_launch();
  SPTS_CUDA_TRY(cudaGetLastError());
  return SPTS_OK;
}

}  // namespace spts
