// rowops.cu -- HBM-bound row kernels of the layer: RMSNorm (with optional
// row gather) to bf16, in-place rotate-half RoPE, 16-byte row gather, the
// synthetic salient-key injection, and the per-group score reduction.
//
// All of these move whole rows with 16-byte vector accesses, one warp per
// row, so a warp touches 512 contiguous bytes per instruction.
#include "host.hpp"
#include "rowops.cuh"
#include "sm100.cuh"

namespace spts {

// ---------------------------------------------------------------- RMSNorm
// One warp per row; x fp32 [*, D], y bf16.  Row i reads x[rows[i]] (x[i]
// without rows) and writes y[i], or y[rows[i]] when `scatter` (renormalise
// some rows in place).  D % 8 == 0.
__device__ __forceinline__ uint4 norm8(const float (&v)[8], float inv, const __nv_bfloat16 *w, int c) {
  float o[8];
  if (w) {
    uint4 wv = __ldg(reinterpret_cast<const uint4 *>(w) + c);
    const __nv_bfloat16 *wb = reinterpret_cast<const __nv_bfloat16 *>(&wv);
#pragma unroll
    for (int t = 0; t < 8; ++t) o[t] = v[t] * inv * __bfloat162float(wb[t]);
  } else {
#pragma unroll
    for (int t = 0; t < 8; ++t) o[t] = v[t] * inv;
  }
  uint4 r;
  r.x = pack_bf16x2(o[0], o[1]);
  r.y = pack_bf16x2(o[2], o[3]);
  r.z = pack_bf16x2(o[4], o[5]);
  r.w = pack_bf16x2(o[6], o[7]);
  return r;
}

__global__ void __launch_bounds__(256) rmsnorm_rows_kernel(const float *__restrict__ x,
                                                           const int32_t *__restrict__ rows, int64_t m, int D,
                                                           const __nv_bfloat16 *__restrict__ w, float eps,
                                                           __nv_bfloat16 *__restrict__ y, int scatter) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (i >= m) return;
  const int lane = threadIdx.x & 31;
  const int64_t src = rows ? rows[i] : i;
  const int64_t dst = scatter ? src : i;
  const float4 *xr = reinterpret_cast<const float4 *>(x + src * D);
  float ss = 0.f;
  for (int c = lane; c < D / 4; c += 32) {
    float4 v = __ldg(xr + c);
    ss += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float inv = 1.0f / sqrtf(ss / static_cast<float>(D) + eps);
  uint4 *yr = reinterpret_cast<uint4 *>(y + dst * D);
  for (int c = lane; c < D / 8; c += 32) {
    float4 a = __ldg(xr + 2 * c), b = __ldg(xr + 2 * c + 1);
    const float v[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    yr[c] = norm8(v, inv, w, c);
  }
}

// Single-pass variant for D = 256 * V8: each lane keeps its V8 pairs of
// float4 in registers, so the row is read from memory once.
template <int V8>
__global__ void __launch_bounds__(256) rmsnorm_rows_reg_kernel(const float *__restrict__ x,
                                                               const int32_t *__restrict__ rows, int64_t m,
                                                               const __nv_bfloat16 *__restrict__ w, float eps,
                                                               __nv_bfloat16 *__restrict__ y, int scatter) {
  constexpr int D = 256 * V8;
  const int64_t i = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (i >= m) return;
  const int lane = threadIdx.x & 31;
  const int64_t src = rows ? rows[i] : i;
  const int64_t dst = scatter ? src : i;
  const float4 *xr = reinterpret_cast<const float4 *>(x + src * D);
  float4 a[V8], b[V8];
#pragma unroll
  for (int t = 0; t < V8; ++t) {
    const int c = lane + 32 * t;  // 8-element column group
    a[t] = __ldg(xr + 2 * c);
    b[t] = __ldg(xr + 2 * c + 1);
  }
  float ss[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int t = 0; t < V8; ++t) {
    ss[0] += a[t].x * a[t].x + b[t].x * b[t].x;
    ss[1] += a[t].y * a[t].y + b[t].y * b[t].y;
    ss[2] += a[t].z * a[t].z + b[t].z * b[t].z;
    ss[3] += a[t].w * a[t].w + b[t].w * b[t].w;
  }
  float s = (ss[0] + ss[1]) + (ss[2] + ss[3]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  const float inv = 1.0f / sqrtf(s / static_cast<float>(D) + eps);
  uint4 *yr = reinterpret_cast<uint4 *>(y + dst * D);
#pragma unroll
  for (int t = 0; t < V8; ++t) {
    const int c = lane + 32 * t;
    const float v[8] = {a[t].x, a[t].y, a[t].z, a[t].w, b[t].x, b[t].y, b[t].z, b[t].w};
    yr[c] = norm8(v, inv, w, c);
  }
}

spts_status launch_rmsnorm_rows(const float *x, const int32_t *rows, int64_t m, int D, const void *w, float eps,
                                void *y, cudaStream_t s, bool scatter) {
  if (m == 0) return SPTS_OK;
  const unsigned blocks = static_cast<unsigned>((m + 7) / 8);
  const __nv_bfloat16 *wb = static_cast<const __nv_bfloat16 *>(w);
  __nv_bfloat16 *yb = static_cast<__nv_bfloat16 *>(y);
  const int sc = scatter ? 1 : 0;
  if (D == 4096)
    rmsnorm_rows_reg_kernel<16><<<blocks, 256, 0, s>>>(x, rows, m, wb, eps, yb, sc);
  else if (D == 1024)
    rmsnorm_rows_reg_kernel<4><<<blocks, 256, 0, s>>>(x, rows, m, wb, eps, yb, sc);
  else
    rmsnorm_rows_kernel<<<blocks, 256, 0, s>>>(x, rows, m, D, wb, eps, yb, sc);
  note_launch();
  SPTS_CUDA_TRY(cudaGetLastError());
  return SPTS_OK;
}

// ---------------------------------------------------------------- RoPE
// Rotate-half RoPE with the angles of rope_cos_sin (reduced in turns, error
// ~1e-6).  One thread per (row, pair i), looping over the heads.
__global__ void rope_kernel(__nv_bfloat16 *__restrict__ x, int64_t m, int H, int d,
                            const int32_t *__restrict__ pos, RopeFreqs f) {
  const int half = d / 2;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= m * half) return;
  const int64_t row = t / half;
  const int i = static_cast<int>(t % half);
  float c, s;
  rope_cos_sin(pos[row], f, i, &c, &s);
  __nv_bfloat16 *xr = x + row * static_cast<int64_t>(H) * d;
  for (int h = 0; h < H; ++h) {
    const float x1 = __bfloat162float(xr[h * d + i]);
    const float x2 = __bfloat162float(xr[h * d + i + half]);
    xr[h * d + i] = __float2bfloat16_rn(x1 * c - x2 * s);
    xr[h * d + i + half] = __float2bfloat16_rn(x2 * c + x1 * s);
  }
}

void fill_rope_freqs(RopeFreqs *f, int d, double theta) {
  for (int i = 0; i < d / 2 && i < 128; ++i) {
    f->inv_freq[i] = pow(theta, -2.0 * i / d);
    const double g = f->inv_freq[i] / 6.283185307179586476925286766559;
    f->turn_hi[i] = static_cast<float>(g);
    f->turn_lo[i] = static_cast<float>(g - static_cast<double>(f->turn_hi[i]));
  }
}

spts_status launch_rope(void *x, int64_t m, int H, int d, const int32_t *pos, double theta, cudaStream_t s) {
  if (m == 0) return SPTS_OK;
  RopeFreqs f;
  fill_rope_freqs(&f, d, theta);
  const int64_t n = m * (d / 2);
  rope_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, s>>>(static_cast<__nv_bfloat16 *>(x), m, H, d,
                                                                      pos, f);
  note_launch();
  SPTS_CUDA_TRY(cudaGetLastError());
  return SPTS_OK;
}

// ---------------------------------------------------------------- gather
// One warp per destination row, 16-byte copies.  Rows outside [0, n_src)
// are skipped and reported in the status word.
__global__ void __launch_bounds__(256) gather_rows_kernel(const uint4 *__restrict__ src, int64_t n_src,
                                                          const int32_t *__restrict__ rows, int64_t m,
                                                          int64_t vec_per_row, uint4 *__restrict__ dst,
                                                          const int32_t *__restrict__ pos_in,
                                                          int32_t *__restrict__ pos_out, uint32_t *status) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (i >= m) return;
  const int lane = threadIdx.x & 31;
  const int32_t r = rows[i];
  if (r < 0 || r >= n_src) {
    if (lane == 0) raise_status(status, SPTS_DEV_BADINDEX, 0x61u, static_cast<uint32_t>(r));
    return;
  }
  const uint4 *s = src + static_cast<int64_t>(r) * vec_per_row;
  uint4 *d = dst + i * vec_per_row;
  for (int64_t c = lane; c < vec_per_row; c += 32) d[c] = __ldg(s + c);
  if (pos_out && lane == 0) pos_out[i] = pos_in[r];
}

spts_status launch_gather_rows(const void *src, int64_t n_src, const int32_t *rows, int64_t m, int64_t row_bytes,
                               void *dst, const int32_t *pos_in, int32_t *pos_out, uint32_t *status,
                               cudaStream_t s) {
  if (m == 0) return SPTS_OK;
  gather_rows_kernel<<<static_cast<unsigned>((m + 7) / 8), 256, 0, s>>>(
      static_cast<const uint4 *>(src), n_src, rows, m, row_bytes / 16, static_cast<uint4 *>(dst), pos_in, pos_out,
      status);
  note_launch();
  SPTS_CUDA_TRY(cudaGetLastError());
  return SPTS_OK;
}

spts_status preload_gather_rows() {
  cudaFuncAttributes a;
  SPTS_CUDA_TRY(cudaFuncGetAttributes(&a, gather_rows_kernel));
  return SPTS_OK;
}

// ---------------------------------------------------------------- salience
// Synthetic-workload step (not SPTS): K[rows[t], g] += shift * unit(mean of
// the group's probe queries).  Blocks (KV head, chunk of SAL_ROWS rows) of
// SAL_THREADS threads = S slices of d threads (d a power of two <= 1024).
// Each block recomputes the group mean: slice s sums the query vectors
// s, s + S, ... with eight loads in flight per thread, in fp64, where the sum
// of bf16 values is exact, so the slice order does not change it.  Slice s
// then updates rows t_begin + s, + S, ... (rows must be distinct).
constexpr int SAL_ROWS = 64;
constexpr int SAL_THREADS = 1024;
constexpr int SAL_BATCH = 8;

__global__ void __launch_bounds__(SAL_THREADS)
    inject_salience_kernel(__nv_bfloat16 *__restrict__ k, int64_t Nc, const __nv_bfloat16 *__restrict__ q, int P,
                           int Hq, int Hkv, int d, const int32_t *__restrict__ rows, int64_t n_rows, float shift,
                           uint32_t *status) {
  extern __shared__ double part[];                          // [S][d] partial sums
  float *red = reinterpret_cast<float *>(part + SAL_THREADS);  // [d] squares, then [d] means
  float *meanv = red + d;
  const int g = blockIdx.x, G = Hq / Hkv, S = SAL_THREADS / d;
  const int i = static_cast<int>(threadIdx.x) % d, sl = static_cast<int>(threadIdx.x) / d;
  const int n = P * G;
  double acc = 0.0;
  for (int pg0 = sl; pg0 < n; pg0 += SAL_BATCH * S) {
    float v[SAL_BATCH];
#pragma unroll
    for (int u = 0; u < SAL_BATCH; ++u) {
      const int pg = pg0 + u * S;
      v[u] = pg < n ? __bfloat162float(q[(static_cast<int64_t>(pg / G) * Hq + g * G + pg % G) * d + i]) : 0.f;
    }
#pragma unroll
    for (int u = 0; u < SAL_BATCH; ++u) acc += v[u];
  }
  part[sl * d + i] = acc;
  __syncthreads();
  if (sl == 0) {
    double t = 0.0;
    for (int j = 0; j < S; ++j) t += part[j * d + i];
    const float mean = static_cast<float>(t / n);
    meanv[i] = mean;
    red[i] = mean * mean;
  }
  __syncthreads();
  for (int o = d / 2; o > 0; o >>= 1) {
    if (sl == 0 && i < o) red[i] += red[i + o];
    __syncthreads();
  }
  const float u = meanv[i] / sqrtf(red[0]);
  const int64_t t_begin = static_cast<int64_t>(blockIdx.y) * SAL_ROWS;
  const int64_t t_end = t_begin + SAL_ROWS < n_rows ? t_begin + SAL_ROWS : n_rows;
  // SAL_BATCH rows per pass: their index and element loads are all in flight
  // together instead of one dependent round trip per row
  for (int64_t t0 = t_begin + sl; t0 < t_end; t0 += static_cast<int64_t>(SAL_BATCH) * S) {
    int32_t row[SAL_BATCH];
    float v[SAL_BATCH];
#pragma unroll
    for (int j = 0; j < SAL_BATCH; ++j) row[j] = t0 + j * S < t_end ? rows[t0 + j * S] : -1;
#pragma unroll
    for (int j = 0; j < SAL_BATCH; ++j) {
      const bool ok = row[j] >= 0 && row[j] < Nc;
      v[j] = ok ? __bfloat162float(k[(static_cast<int64_t>(row[j]) * Hkv + g) * d + i]) : 0.f;
    }
#pragma unroll
    for (int j = 0; j < SAL_BATCH; ++j) {
      if (t0 + j * S >= t_end) break;
      if (row[j] < 0 || row[j] >= Nc) {
        if (i == 0) raise_status(status, SPTS_DEV_BADINDEX, 0x62u, static_cast<uint32_t>(row[j]));
        continue;
      }
      k[(static_cast<int64_t>(row[j]) * Hkv + g) * d + i] = __float2bfloat16_rn(v[j] + shift * u);
    }
  }
}

spts_status launch_inject_salience(void *k, int64_t Nc, const void *q_probe, int P, int Hq, int Hkv, int d,
                                   const int32_t *rows, int64_t n_rows, float shift, uint32_t *status,
                                   cudaStream_t s) {
  if (n_rows == 0) return SPTS_OK;
  const dim3 grid(static_cast<unsigned>(Hkv), static_cast<unsigned>((n_rows + SAL_ROWS - 1) / SAL_ROWS));
  const size_t smem = SAL_THREADS * sizeof(double) + 2 * static_cast<size_t>(d) * sizeof(float);
  inject_salience_kernel<<<grid, SAL_THREADS, smem, s>>>(static_cast<__nv_bfloat16 *>(k), Nc,
                                                         static_cast<const __nv_bfloat16 *>(q_probe), P, Hq, Hkv,
                                                         d, rows, n_rows, shift, status);
  note_launch();
  SPTS_CUDA_TRY(cudaGetLastError());
  return SPTS_OK;
}

// ---------------------------------------------------------------- group sum
// s[j] = sum_g group[g][j], fixed order (deterministic).
__global__ void sum_groups_kernel(const float *__restrict__ group, int G, int64_t n, float *__restrict__ s) {
  const int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (j >= n) return;
  float acc = 0.f;
  for (int g = 0; g < G; ++g) acc += group[g * n + j];
  s[j] = acc;
}

spts_status launch_sum_groups(const float *group, int G, int64_t n, float *s, cudaStream_t st) {
  if (n == 0) return SPTS_OK;
  sum_groups_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, st>>>(group, G, n, s);
  note_launch();
  SPTS_CUDA_TRY(cudaGetLastError());
  return SPTS_OK;
}

}  // namespace spts

namespace spts {

// dst[i] = i.
__global__ void iota_i32_kernel(int32_t *__restrict__ dst, int64_t n) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i < n) dst[i] = static_cast<int32_t>(i);
}

spts_status launch_iota_i32(int32_t *dst, int64_t n, cudaStream_t s) {
  if (n == 0) return SPTS_OK;
  iota_i32_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, s>>>(dst, n);
  note_launch();
  SPTS_CUDA_TRY(cudaGetLastError());
  return SPTS_OK;
}

// dst[i] = src[idx[i]] for int32 vectors (positions of the selected rows).
__global__ void gather_i32_kernel(const int32_t *__restrict__ src, const int32_t *__restrict__ idx, int64_t m,
                                  int32_t *__restrict__ dst) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i < m) dst[i] = src[idx[i]];
}

spts_status launch_gather_i32(const int32_t *src, const int32_t *idx, int64_t m, int32_t *dst, cudaStream_t s) {
  if (m == 0) return SPTS_OK;
  gather_i32_kernel<<<static_cast<unsigned>((m + 255) / 256), 256, 0, s>>>(src, idx, m, dst);
  note_launch();
  SPTS_CUDA_TRY(cudaGetLastError());
  return SPTS_OK;
}

// ---------------------------------------------------------------- bf16 residual boundary
// dst[i] = float(src[i]) for n elements (n % 8 == 0), 16-byte loads.
__global__ void bf16_to_f32_kernel(const uint4 *__restrict__ src, int64_t n8, float4 *__restrict__ dst) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8; i += stride) {
    const uint4 v = src[i];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    float f[8];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      f[2 * q] = __uint_as_float(w[q] << 16);
      f[2 * q + 1] = __uint_as_float(w[q] & 0xFFFF0000u);
    }
    dst[2 * i] = make_float4(f[0], f[1], f[2], f[3]);
    dst[2 * i + 1] = make_float4(f[4], f[5], f[6], f[7]);
  }
}

// dst[rows[t]] = bf16(src[rows[t]]) (round to nearest even) for t < m, rows
// of D elements (D % 8 == 0): one warp per row, 16-byte stores.
__global__ void rows_f32_to_bf16_kernel(const float4 *__restrict__ src, const int32_t *__restrict__ rows, int64_t m,
                                        int64_t n_rows, int d8, uint4 *__restrict__ dst, uint32_t *status) {
  const int64_t t = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (t >= m) return;
  const int64_t r = rows[t];
  if (r < 0 || r >= n_rows) {
    if (lane == 0) raise_status(status, SPTS_DEV_BADINDEX, 0x61u, static_cast<uint32_t>(r));
    return;
  }
  for (int c = lane; c < d8; c += 32) {
    const float4 a = src[(r * d8 + c) * 2], b = src[(r * d8 + c) * 2 + 1];
    dst[r * d8 + c] = make_uint4(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w), pack_bf16x2(b.x, b.y),
                                 pack_bf16x2(b.z, b.w));
  }
}

spts_status launch_bf16_to_f32(const void *src, int64_t n, float *dst, cudaStream_t s) {
  if (n == 0) return SPTS_OK;
  const int64_t n8 = n / 8;
  const int64_t blocks = std::min<int64_t>((n8 + 255) / 256, static_cast<int64_t>(num_sms()) * 8);
  bf16_to_f32_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(static_cast<const uint4 *>(src), n8,
                                                                      reinterpret_cast<float4 *>(dst));
  note_launch();
  SPTS_CUDA_TRY(cudaGetLastError());
  return SPTS_OK;
}

spts_status launch_rows_f32_to_bf16(const float *src, const int32_t *rows, int64_t m, int64_t n_rows, int D,
                                    void *dst, uint32_t *status, cudaStream_t s) {
  if (m == 0) return SPTS_OK;
  rows_f32_to_bf16_kernel<<<static_cast<unsigned>((m + 7) / 8), 256, 0, s>>>(
      reinterpret_cast<const float4 *>(src), rows, m, n_rows, D / 8, static_cast<uint4 *>(dst), status);
  note_launch();
  SPTS_CUDA_TRY(cudaGetLastError());
  return SPTS_OK;
}

// ---------------------------------------------------------------- test hook
// y[i] = exp2_poly2(x[i]): the FMA-pipe exp2 of the reduced-attention softmax, on its own.
__global__ void exp2_poly_kernel(const float *__restrict__ x, int64_t n, float *__restrict__ y) {
  const int64_t i = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) * 2;
  if (i >= n) return;
  const float a = x[i], b = i + 1 < n ? x[i + 1] : x[i];
  float e0, e1;
  exp2_poly2(f2pack(a, b), e0, e1);
  y[i] = e0;
  if (i + 1 < n) y[i + 1] = e1;
}

spts_status launch_exp2_poly(const float *x, int64_t n, float *y, cudaStream_t s) {
  if (n == 0) return SPTS_OK;
  exp2_poly_kernel<<<static_cast<unsigned>((n + 511) / 512), 256, 0, s>>>(x, n, y);
  note_launch();
  SPTS_CUDA_TRY(cudaGetLastError());
  return SPTS_OK;
}

}  // namespace spts
