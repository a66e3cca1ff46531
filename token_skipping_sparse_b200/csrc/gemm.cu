// gemm.cu -- bf16 tensor-core GEMM acc = A W^T on sm_100a with fused epilogues.
//
// This is the projection engine of the SPTS layer: K/V (+RoPE) for every
// candidate, Q for the probe rows and for the selected rows, the O
// projection added into the residual at the selected rows, and the reduced
// SwiGLU FFN (gate/up with the SwiGLU product, down added into the residual).
//
// Design for M <= 128 (one CTA per SM, persistent over 128 x 256 output tiles;
// larger M uses the two-SM 256 x 256 tiles further down):
//   warp 0      TMA producer: A tile 128x64 and B tile 256x64 per stage into
//               a 4-stage ring of 128-byte-swizzled shared memory;
//   warp 1      MMA issuer: the warp runs the loop, one elected lane
//               issues tcgen05.mma (M=128, N=256, K=16) into one of two TMEM
//               accumulators (2 x 256 columns);
//   warps 2..5  epilogue: tcgen05.ld of the accumulator rows (warp w reads
//               TMEM lanes 32*(w%4)..+31), then the fused epilogue and the
//               global stores, overlapping the next tile's main loop.
// Tiles are visited in groups of 16 M-tiles (M fastest inside a group) so a
// wave of 148 CTAs shares both operands through L2.
// Every barrier wait is bounded (see sm100.cuh).
#include "host.hpp"
#include "rowops.cuh"
#include "sm100.cuh"

namespace spts {
namespace {

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;                 // 16 KB
constexpr int B_BYTES = BN * BK * 2;                 // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;       // 48 KB
constexpr int GROUP_M = 16;
constexpr int THREADS = 192;
constexpr uint32_t TMEM_COLS = 512;
// Scatter-add staging: per epilogue warp 32 rows x 32 fp32, rows padded to
// 36 words so that the row-per-thread writes and the row-segment reads of
// 16-byte vectors are both free of bank conflicts.
constexpr int STG_STRIDE = 36;
constexpr int STG_BYTES = 4 * 32 * STG_STRIDE * 4;   // 18 KB
constexpr size_t SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + 256 + STG_BYTES;

struct Params {
  int M, N, K;         // N: output columns of W (for SWIGLU: of W_gate and of W_up each)
  int tiles_m, tiles_n;
  int split_from;      // two-SM tiles from this index on run as two 128-column halves
  void *out;
  const int32_t *rows;
  const int32_t *row_pos;
  uint32_t *status;
  uint64_t wait_ns;
  RopeFreqs freqs;
};

__device__ __forceinline__ void tile_coords(int t, int tiles_m, int tiles_n, int &tm, int &tn) {
  const int per_group = GROUP_M * tiles_n;
  const int grp = t / per_group;
  const int first_m = grp * GROUP_M;
  const int gm = min(GROUP_M, tiles_m - first_m);
  const int r = t - grp * per_group;
  tm = first_m + r % gm;
  tn = r / gm;
}

__device__ __forceinline__ float silu(float g) { return g / (1.0f + __expf(-g)); }

__device__ __forceinline__ void store_bf16x32(__nv_bfloat16 *dst, const float *v) {
  uint4 *d4 = reinterpret_cast<uint4 *>(dst);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint4 o;
    o.x = pack_bf16x2(v[8 * q + 0], v[8 * q + 1]);
    o.y = pack_bf16x2(v[8 * q + 2], v[8 * q + 3]);
    o.z = pack_bf16x2(v[8 * q + 4], v[8 * q + 5]);
    o.w = pack_bf16x2(v[8 * q + 6], v[8 * q + 7]);
    d4[q] = o;
  }
}


// Fused epilogue of one accumulator tile of `width` columns (256, or 128
// for half a tile) for the 32 rows this warp owns: `tbase` addresses the
// warp's TMEM lanes at the tile's first column; `row` is this thread's
// output row, `col0` the output column of the tile's first result column.
template <int EPI>
__device__ __forceinline__ void epilogue_rows(const Params &p, uint32_t tbase, int64_t row, bool live, int col0,
                                              int width, float *stg) {
  if (EPI == SPTS_EPI_STORE) {
    __nv_bfloat16 *out = static_cast<__nv_bfloat16 *>(p.out);
#pragma unroll 1
    for (int c = 0; c < width / 32; ++c) {
      uint32_t r[32];
      tmem_ld32(tbase + c * 32, r);
      tmem_ld_wait();
      if (live) store_bf16x32(out + row * p.N + col0 + c * 32, reinterpret_cast<float *>(r));
    }
  } else if (EPI == SPTS_EPI_ROPE) {
    __nv_bfloat16 *out = static_cast<__nv_bfloat16 *>(p.out);
    const int32_t pos = live ? p.row_pos[row] : 0;
#pragma unroll 1
    for (int c = 0; c < 2; ++c) {               // pairs i in [32c, 32c+32), partner i+64
      // one angle per pair, shared by the tile's heads (same row position)
      float cs[32], sn[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) rope_cos_sin(pos, p.freqs, c * 32 + i, &cs[i], &sn[i]);
#pragma unroll 1
      for (int hc = 0; hc < width / 128; ++hc) {   // heads of 128 columns in this tile
        uint32_t lo[32], hi[32];
        tmem_ld32(tbase + hc * 128 + c * 32, lo);
        tmem_ld32(tbase + hc * 128 + 64 + c * 32, hi);
        tmem_ld_wait();
        float yl[32], yh[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float xl = __uint_as_float(lo[i]), xh = __uint_as_float(hi[i]);
          yl[i] = xl * cs[i] - xh * sn[i];
          yh[i] = xh * cs[i] + xl * sn[i];
        }
        if (live) {
          __nv_bfloat16 *o = out + row * p.N + col0 + hc * 128;
          store_bf16x32(o + c * 32, yl);
          store_bf16x32(o + 64 + c * 32, yh);
        }
      }
    }
  } else if (EPI == SPTS_EPI_SWIGLU) {
    __nv_bfloat16 *out = static_cast<__nv_bfloat16 *>(p.out);
#pragma unroll 1
    for (int c = 0; c < width / 64; ++c) {      // gate in the first half of the columns, up in the second
      uint32_t g[32], u[32];
      tmem_ld32(tbase + c * 32, g);
      tmem_ld32(tbase + width / 2 + c * 32, u);
      tmem_ld_wait();
      float y[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) y[i] = silu(__uint_as_float(g[i])) * __uint_as_float(u[i]);
      if (live) store_bf16x32(out + row * p.N + col0 + c * 32, y);
    }
  } else {  // SCATTER_ADD into fp32 rows (unique rows): each 32-column chunk of the warp's 32 rows goes
           // through shared memory so that 8 lanes update one row's 128 contiguous bytes: coalesced
           // loads and stores instead of 32 scattered half-sector reductions per instruction
    float *out = static_cast<float *>(p.out);
    const int lane = threadIdx.x & 31;
    const int64_t orow = live ? p.rows[row] : -1;
    int64_t dst[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) dst[i] = __shfl_sync(0xffffffffu, orow, 4 * i + (lane >> 3));
    float4 *srow = reinterpret_cast<float4 *>(stg + lane * STG_STRIDE);
#pragma unroll 1
    for (int c = 0; c < width / 32; ++c) {
      uint32_t r[32];
      tmem_ld32(tbase + c * 32, r);
      tmem_ld_wait();
#pragma unroll
      for (int q = 0; q < 8; ++q)
        srow[q] = make_float4(__uint_as_float(r[4 * q]), __uint_as_float(r[4 * q + 1]),
                              __uint_as_float(r[4 * q + 2]), __uint_as_float(r[4 * q + 3]));
      __syncwarp();
      float4 hv[8];
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (dst[i] >= 0)
          hv[i] = reinterpret_cast<const float4 *>(out + dst[i] * p.N + col0 + c * 32)[lane & 7];
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (dst[i] >= 0) {
          const float4 v = reinterpret_cast<const float4 *>(stg + (4 * i + (lane >> 3)) * STG_STRIDE)[lane & 7];
          hv[i].x += v.x;
          hv[i].y += v.y;
          hv[i].z += v.z;
          hv[i].w += v.w;
          reinterpret_cast<float4 *>(out + dst[i] * p.N + col0 + c * 32)[lane & 7] = hv[i];
        }
      __syncwarp();
    }
  }
}

template <int EPI>
__global__ void __launch_bounds__(THREADS, 1)
    gemm_bf16_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmB2, const __grid_constant__ Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sA = smem;
  uint8_t *sB = smem + STAGES * A_BYTES;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + STAGES * STAGE_BYTES);
  uint64_t *full = bars, *empty = bars + STAGES, *tfull = bars + 2 * STAGES, *tempty = tfull + 2,
           *drain = tempty + 2;
  uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(drain + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 128);
    }
    mbar_init(drain, 1);
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
  const int tiles = p.tiles_m * p.tiles_n;
  const int kblocks = p.K / BK;

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmB);
      if (EPI == SPTS_EPI_SWIGLU) tma_prefetch_desc(&tmB2);
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, issued_phase = 0;
      for (int t = blockIdx.x; t < tiles && !*abort_flag; t += gridDim.x) {
        int tm, tn;
        tile_coords(t, p.tiles_m, p.tiles_n, tm, tn);
        const int m0 = tm * BM;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, p.status, p.wait_ns, 0x11u)) break;
          mbar_arrive_expect_tx(&full[stage], STAGE_BYTES);
          uint8_t *a_dst = sA + stage * A_BYTES;
          uint8_t *b_dst = sB + stage * B_BYTES;
          tma_load_2d(a_dst, &tmA, &full[stage], kb * BK, m0);
          if (EPI == SPTS_EPI_SWIGLU) {
            tma_load_2d(b_dst, &tmB, &full[stage], kb * BK, tn * 128);
            tma_load_2d(b_dst + B_BYTES / 2, &tmB2, &full[stage], kb * BK, tn * 128);
          } else {
            tma_load_2d(b_dst, &tmB, &full[stage], kb * BK, tn * BN);
            tma_load_2d(b_dst + B_BYTES / 2, &tmB, &full[stage], kb * BK, tn * BN + 128);
          }
          issued_mask |= 1u << stage;
          issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (*abort_flag) {
        // let the copies already in flight land before the CTA exits
        for (int s = 0; s < STAGES; ++s)
          if (issued_mask & (1u << s)) mbar_drain(&full[s], (issued_phase >> s) & 1u, p.status);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    {  // the whole warp runs the issue loop; one elected lane issues each MMA and commit
      constexpr uint32_t idesc = idesc_bf16_f32(BM, BN, 0, 0);
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x, ++local) {
        const int acc = local & 1;
        const uint32_t acc_phase = (local >> 1) & 1;
        if (!__all_sync(0xffffffffu,
                        mbar_wait(&tempty[acc], acc_phase ^ 1u, abort_flag, p.status, p.wait_ns, 0x12u)))
          break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!__all_sync(0xffffffffu, mbar_wait(&full[stage], phase, abort_flag, p.status, p.wait_ns, 0x13u))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t adesc = sdesc_k_sw128(smem_u32(sA + stage * A_BYTES));
          const uint64_t bdesc = sdesc_k_sw128(smem_u32(sB + stage * B_BYTES));
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            mma_bf16_ss_w(d_tmem, adesc + 2 * kk, bdesc + 2 * kk, idesc, (kb | kk) != 0);
          tc_commit_w(&empty[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (ok) tc_commit_w(&tfull[acc]);
      }
      // every MMA issued so far must finish before TMEM is released
      tc_commit_w(drain);
      mbar_drain(drain, 0, p.status);
    }
    __syncwarp();
  } else {
    // epilogue warps 2..5 -> TMEM lane quadrant warp % 4
    const int quad = warp & 3;
    const int row_in_tile = quad * 32 + lane;
    float *stg = reinterpret_cast<float *>(smem + STAGES * STAGE_BYTES + 256) + (warp - 2) * 32 * STG_STRIDE;
    int local = 0;
    for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++local) {
      const int acc = local & 1;
      const uint32_t acc_phase = (local >> 1) & 1;
      const bool ok = mbar_wait(&tfull[acc], acc_phase, abort_flag, p.status, p.wait_ns, 0x14u);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      int tm, tn;
      tile_coords(t, p.tiles_m, p.tiles_n, tm, tn);
      const int64_t row = static_cast<int64_t>(tm) * BM + row_in_tile;
      const bool live = row < p.M;
      const uint32_t tbase = tmem_addr(tmem_base, quad * 32, acc * BN);
      epilogue_rows<EPI>(p, tbase, row, live, EPI == SPTS_EPI_SWIGLU ? tn * 128 : tn * BN, BN, stg);
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

template <int EPI>
spts_status launch_epi(const GemmArgs &g, const CUtensorMap &ta, const CUtensorMap &tb, const CUtensorMap &tb2,
                       Params &p, cudaStream_t s) {
  SPTS_CUDA_TRY(cudaFuncSetAttribute(gemm_bf16_kernel<EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     static_cast<int>(SMEM_BYTES)));
  const int tiles = p.tiles_m * p.tiles_n;
  const int grid = tiles < num_sms() ? tiles : num_sms();
  gemm_bf16_kernel<EPI><<<grid, THREADS, SMEM_BYTES, s>>>(ta, tb, tb2, p);
  note_launch();
  SPTS_CUDA_TRY(cudaGetLastError());
  return SPTS_OK;
}


// ---------------------------------------------------------------- two-SM tiles
// A (2,1,1) cluster computes a 256 x 256 tile with cta_group::2 MMAs
// (M = 256).  CTA r loads rows [128 r, 128 r + 128) of the A tile and rows
// [128 r, 128 r + 128) of the B tile (accumulator columns [128 r, 128 r +
// 128); for SWIGLU CTA 0 loads W_gate, CTA 1 W_up) into its own 6-stage ring;
// its TMEM holds its 128 output rows x 256 columns.  Each SM streams half of
// B: per K = 16 step 4 KB of A and 4 KB of B from its shared memory instead of
// 4 KB of A and 8 KB of B.
//   warp 0      TMA in both CTAs; every copy completes on CTA 0's full[]
//               barrier, whose expected bytes CTA 0 posts for both halves;
//   warp 1      CTA 0: MMA issuer for the pair, warp-wide with one elected
//               lane issuing (stage and accumulator releases are commits
//               multicast to both CTAs);
//   warps 2..5  epilogue of this CTA's rows; they release an accumulator on
//               CTA 0's tempty[] barrier (128 arrivals from each CTA).
// When the last round of tiles would keep at most half of the pairs busy,
// those tiles run as two 128-column halves each (N = 128 MMAs, each CTA
// supplying 64 rows of B), so the round takes half as long.
// Loads are plain tile loads (no multicast): each CTA reads only its own
// operand halves.  On exit the two CTAs reconcile the copies each issued per
// stage so that CTA 0 can wait for every copy still in flight (a timeout may
// have stopped one producer before the other).
constexpr int STAGES2 = 6;
constexpr int HALF_BYTES = 128 * BK * 2;       // 16 KB: 128 rows x 64 bf16
constexpr int STAGE2_BYTES = 2 * HALF_BYTES;   // one CTA's A half + B half
constexpr int GROUP_M2 = 8;                    // 256-row tiles per raster group
constexpr size_t SMEM2_BYTES = 1024 + STAGES2 * STAGE2_BYTES + 256 + STG_BYTES;

__device__ __forceinline__ void tile_coords2(int t, int tiles_m2, int tiles_n, int &tm, int &tn) {
  const int per_group = GROUP_M2 * tiles_n;
  const int grp = t / per_group;
  const int first_m = grp * GROUP_M2;
  const int gm = min(GROUP_M2, tiles_m2 - first_m);
  const int r = t - grp * per_group;
  tm = first_m + r % gm;
  tn = r / gm;
}

// Unit u of a CTA pair's schedule: a whole 256-column tile, or, from tile
// split_from on (the last round of tiles when it fills at most half of the
// pairs), one of its two 128-column halves (half = 0 or 1; -1: whole tile).
__device__ __forceinline__ void unit_coords2(int u, int split_from, int tiles_m2, int tiles_n, int &tm, int &tn,
                                             int &half) {
  int t = u;
  half = -1;
  if (u >= split_from) {
    t = split_from + ((u - split_from) >> 1);
    half = (u - split_from) & 1;
  }
  tile_coords2(t, tiles_m2, tiles_n, tm, tn);
}

template <int EPI>
__global__ void __launch_bounds__(THREADS, 1)
    gemm2_bf16_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                      const __grid_constant__ CUtensorMap tmB2, const __grid_constant__ Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sA = smem;                          // STAGES2 x A half
  uint8_t *sB = smem + STAGES2 * HALF_BYTES;   // STAGES2 x B half
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + STAGES2 * STAGE2_BYTES);
  uint64_t *full = bars, *empty = bars + STAGES2, *tfull = bars + 2 * STAGES2, *tempty = tfull + 2,
           *drain = tempty + 2;
  uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(drain + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);
  uint32_t *rounds = tmem_holder + 2;                // copies this CTA issued per stage
  uint32_t *peer_rounds = rounds + STAGES2;          // CTA 0: the same counts of CTA 1

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const int pair = static_cast<int>(blockIdx.x) >> 1, n_pairs = static_cast<int>(gridDim.x) >> 1;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES2; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      rounds[s] = 0;
      peer_rounds[s] = 0;
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 256);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc_pair(tmem_holder, TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // the peer's barriers exist before any copy or arrival targets them
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const int tiles_m2 = (p.tiles_m + 1) >> 1;
  const int tiles = tiles_m2 * p.tiles_n;
  const int units = p.split_from + 2 * (tiles - p.split_from);
  const int kblocks = p.K / BK;

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmB);
      if (EPI == SPTS_EPI_SWIGLU) tma_prefetch_desc(&tmB2);
      const CUtensorMap *mb = (EPI == SPTS_EPI_SWIGLU && rank == 1) ? &tmB2 : &tmB;
      int stage = 0;
      uint32_t phase = 0;
      for (int t = pair; t < units && !*abort_flag; t += n_pairs) {
        int tm, tn, half;
        unit_coords2(t, p.split_from, tiles_m2, p.tiles_n, tm, tn, half);
        const int a_row = tm * 256 + static_cast<int>(rank) * 128;
        // each CTA supplies half of the tile's N rows of B (a half tile: 64
        // of the 128 rows its box loads; the rest is not read)
        const int b_row = EPI == SPTS_EPI_SWIGLU ? tn * 128 + (half < 0 ? 0 : half * 64)
                          : half < 0               ? tn * BN + static_cast<int>(rank) * 128
                                                   : tn * BN + half * 128 + static_cast<int>(rank) * 64;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, p.status, p.wait_ns, 0x31u)) break;
          if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * STAGE2_BYTES);
          tma_load_2d_pair(sA + stage * HALF_BYTES, &tmA, &full[stage], kb * BK, a_row);
          tma_load_2d_pair(sB + stage * HALF_BYTES, mb, &full[stage], kb * BK, b_row);
          rounds[stage] += 1;
          if (++stage == STAGES2) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (rank == 0) {  // the whole warp runs the issue loop; one elected lane issues each MMA and commit
      constexpr uint32_t idesc_full = idesc_bf16_f32(256, BN, 0, 0);
      constexpr uint32_t idesc_half = idesc_bf16_f32(256, BN / 2, 0, 0);
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      bool ok = true;
      for (int t = pair; t < units && ok; t += n_pairs, ++local) {
        const uint32_t idesc = t < p.split_from ? idesc_full : idesc_half;
        const int acc = local & 1;
        const uint32_t acc_phase = (local >> 1) & 1;
        if (!__all_sync(0xffffffffu,
                        mbar_wait_cluster(&tempty[acc], acc_phase ^ 1u, abort_flag, p.status, p.wait_ns, 0x32u)))
          break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!__all_sync(0xffffffffu, mbar_wait(&full[stage], phase, abort_flag, p.status, p.wait_ns, 0x33u))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t adesc = sdesc_k_sw128(smem_u32(sA + stage * HALF_BYTES));
          const uint64_t bdesc = sdesc_k_sw128(smem_u32(sB + stage * HALF_BYTES));
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            mma2_bf16_ss_w(d_tmem, adesc + 2 * kk, bdesc + 2 * kk, idesc, (kb | kk) != 0);
          tc2_commit_both_w(&empty[stage]);
          if (++stage == STAGES2) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (ok) tc2_commit_both_w(&tfull[acc]);
      }
      // every MMA issued so far (they write both CTAs' TMEM) must finish
      tc2_commit_self_w(drain);
      mbar_drain(drain, 0, p.status);
    }
    __syncwarp();
  } else {
    const int quad = warp & 3;
    const int row_in_tile = quad * 32 + lane;
    float *stg = reinterpret_cast<float *>(smem + STAGES2 * STAGE2_BYTES + 256) + (warp - 2) * 32 * STG_STRIDE;
    int local = 0;
    for (int t = pair; t < units; t += n_pairs, ++local) {
      const int acc = local & 1;
      const uint32_t acc_phase = (local >> 1) & 1;
      const bool ok = mbar_wait(&tfull[acc], acc_phase, abort_flag, p.status, p.wait_ns, 0x34u);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      int tm, tn, half;
      unit_coords2(t, p.split_from, tiles_m2, p.tiles_n, tm, tn, half);
      const int64_t row = static_cast<int64_t>(tm) * 256 + rank * 128 + row_in_tile;
      const bool live = row < p.M;
      const uint32_t tbase = tmem_addr(tmem_base, quad * 32, acc * BN);
      const int width = half < 0 ? BN : BN / 2;
      const int col0 = EPI == SPTS_EPI_SWIGLU ? tn * 128 + (half < 0 ? 0 : half * 64)
                                              : tn * BN + (half < 0 ? 0 : half * 128);
      epilogue_rows<EPI>(p, tbase, row, live, col0, width, stg);
      tc_fence_before();
      mbar_arrive_remote(&tempty[acc], 0);
    }
  }
  __syncthreads();
  // Reconcile the copies: CTA 1 reports its per-stage counts to CTA 0, which
  // makes each stage's last phase completable (its own arrival with the
  // expected bytes, or the bytes of a copy the peer never issued) and waits
  // for it.  Without a timeout every copy was consumed and nothing waits.
  if (threadIdx.x == 0 && rank == 1) {
    for (int s = 0; s < STAGES2; ++s)
      asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(cluster_addr(&peer_rounds[s], 0)), "r"(rounds[s])
                   : "memory");
  }
  cluster_sync_all();
  if (threadIdx.x == 0 && rank == 0) {
    for (int s = 0; s < STAGES2; ++s) {
      const uint32_t mine = rounds[s], theirs = peer_rounds[s];
      const uint32_t last = mine > theirs ? mine : theirs;
      if (last == 0) continue;
      if (theirs > mine) mbar_arrive_expect_tx(&full[s], STAGE2_BYTES);  // the peer's half only
      else if (mine > theirs) mbar_complete_tx(&full[s], STAGE2_BYTES);  // the half never issued
      mbar_drain(&full[s], (last - 1) & 1u, p.status);
    }
  }
  cluster_sync_all();  // no CTA leaves while its peer may still signal it or use its TMEM
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

template <int EPI>
spts_status launch_epi2(const CUtensorMap &ta, const CUtensorMap &tb, const CUtensorMap &tb2, Params &p,
                        cudaStream_t s) {
  SPTS_CUDA_TRY(cudaFuncSetAttribute(gemm2_bf16_kernel<EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     static_cast<int>(SMEM2_BYTES)));
  cudaLaunchConfig_t cfg{};
  cfg.blockDim = dim3(THREADS, 1, 1);
  cfg.dynamicSmemBytes = SMEM2_BYTES;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // persistent grid: as many CTA pairs as can be resident at once
  static int resident_pairs[64] = {0};
  int dev = 0;
  SPTS_CUDA_TRY(cudaGetDevice(&dev));
  int &max_pairs = resident_pairs[dev & 63];
  if (max_pairs == 0) {
    cfg.gridDim = dim3(2 * (num_sms() / 2), 1, 1);
    int n = 0;
    SPTS_CUDA_TRY(cudaOccupancyMaxActiveClusters(&n, gemm2_bf16_kernel<EPI>, &cfg));
    max_pairs = n > 0 ? n : 1;
  }
  const int tiles = ((p.tiles_m + 1) >> 1) * p.tiles_n;
  // The last round of tiles, when it would keep at most half of the pairs
  // busy, runs as 128-column halves: one round of half the length.
  const int tail = tiles % max_pairs;
  p.split_from = (tail > 0 && 2 * tail <= max_pairs) ? tiles - tail : tiles;
  const int units = p.split_from + 2 * (tiles - p.split_from);
  const int pairs = units < max_pairs ? units : max_pairs;
  cfg.gridDim = dim3(2 * pairs, 1, 1);
  SPTS_CUDA_TRY(cudaLaunchKernelEx(&cfg, gemm2_bf16_kernel<EPI>, ta, tb, tb2, p));
  note_launch();
  SPTS_CUDA_TRY(cudaGetLastError());
  return SPTS_OK;
}

}  // namespace

spts_status launch_gemm(const GemmArgs &g, cudaStream_t s) {
  if (g.M == 0) return SPTS_OK;
  CUtensorMap ta, tb, tb2;
  SPTS_TRY(tmap_bf16_2d(&ta, g.A, static_cast<uint64_t>(g.M), g.K, g.K, 128));
  SPTS_TRY(tmap_bf16_2d(&tb, g.W, static_cast<uint64_t>(g.N), g.K, g.K, 128));
  if (g.epi == SPTS_EPI_SWIGLU)
    SPTS_TRY(tmap_bf16_2d(&tb2, g.W2, static_cast<uint64_t>(g.N), g.K, g.K, 128));
  else
    tb2 = tb;
  Params p{};
  p.M = static_cast<int>(g.M);
  p.N = g.N;
  p.K = g.K;
  p.tiles_m = static_cast<int>((g.M + BM - 1) / BM);
  p.tiles_n = g.epi == SPTS_EPI_SWIGLU ? g.N / 128 : g.N / BN;
  p.out = g.out;
  p.rows = g.rows;
  p.row_pos = g.row_pos;
  p.status = g.status;
  p.wait_ns = wait_limit_ns();
  if (g.epi == SPTS_EPI_ROPE) fill_rope_freqs(&p.freqs, 128, g.theta);
  if (p.tiles_m > 1) {  // two-SM tiles whenever M spans more than one 128-row tile
    switch (g.epi) {
      case SPTS_EPI_STORE: return launch_epi2<SPTS_EPI_STORE>(ta, tb, tb2, p, s);
      case SPTS_EPI_ROPE: return launch_epi2<SPTS_EPI_ROPE>(ta, tb, tb2, p, s);
      case SPTS_EPI_SWIGLU: return launch_epi2<SPTS_EPI_SWIGLU>(ta, tb, tb2, p, s);
      default: return launch_epi2<SPTS_EPI_SCATTER_ADD>(ta, tb, tb2, p, s);
    }
  }
  switch (g.epi) {
    case SPTS_EPI_STORE: return launch_epi<SPTS_EPI_STORE>(g, ta, tb, tb2, p, s);
    case SPTS_EPI_ROPE: return launch_epi<SPTS_EPI_ROPE>(g, ta, tb, tb2, p, s);
    case SPTS_EPI_SWIGLU: return launch_epi<SPTS_EPI_SWIGLU>(g, ta, tb, tb2, p, s);
    default: return launch_epi<SPTS_EPI_SCATTER_ADD>(g, ta, tb, tb2, p, s);
  }
}

}  // namespace spts
