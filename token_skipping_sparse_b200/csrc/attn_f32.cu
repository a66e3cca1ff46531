// attn_f32.cu -- fp32 CUDA-core paths of PAP and reduced attention.
//
// These serve fp32 data (d = 64 or 128), where a bf16 tensor-core product
// would not meet fp32 accuracy.  They are plain, exact-arithmetic kernels:
//   probe pass 1: one warp per (head, probe) row -> row max and sum of exp;
//   probe pass 2: one thread per key -> sum over heads and probes of the
//                 normalised weight, per KV group, then over groups;
//   attention:    one warp per (query, head), online softmax over the
//                 visible keys, each lane owning d/32 output columns.
#include "host.hpp"
#include "rowops.cuh"

namespace spts {

template <int D>
__device__ __forceinline__ float dot_row(const float *__restrict__ a, const float *__restrict__ b) {
  float acc = 0.f;
#pragma unroll
  for (int t = 0; t < D; t += 4) {
    float4 x = *reinterpret_cast<const float4 *>(a + t);
    float4 y = __ldg(reinterpret_cast<const float4 *>(b + t));
    acc = fmaf(x.x, y.x, acc);
    acc = fmaf(x.y, y.y, acc);
    acc = fmaf(x.z, y.z, acc);
    acc = fmaf(x.w, y.w, acc);
  }
  return acc;
}

// ---------------------------------------------------------------- probe pass 1
template <int D>
__global__ void __launch_bounds__(256) probe_f32_stats(const float *__restrict__ q, const int32_t *__restrict__ qpos,
                                                       int P, const float *__restrict__ k,
                                                       const int32_t *__restrict__ kpos, int64_t Nc, int Hq,
                                                       int Hkv, float scale, float2 *__restrict__ stats) {
  __shared__ __align__(16) float qs[8][D];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * 8 + w;  // row = h * P + p
  const bool live = row < Hq * P;
  const int h = live ? row / P : 0, p = live ? row % P : 0;
  const int g = h / (Hq / Hkv);
  for (int t = lane; t < D; t += 32) qs[w][t] = live ? q[(static_cast<int64_t>(p) * Hq + h) * D + t] * scale : 0.f;
  __syncwarp();
  if (!live) return;
  const int32_t lim = qpos[p];
  float m = -INFINITY, l = 0.f;
  for (int64_t j = lane; j < Nc; j += 32) {
    if (kpos[j] > lim) continue;
    const float x = dot_row<D>(qs[w], k + (j * Hkv + g) * D);
    if (x > m) {
      l = l * expf(m - x) + 1.f;
      m = x;
    } else {
      l += expf(x - m);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
    const float l2 = __shfl_xor_sync(0xffffffffu, l, o);
    const float mm = fmaxf(m, m2);
    l = (m == -INFINITY ? 0.f : l * expf(m - mm)) + (m2 == -INFINITY ? 0.f : l2 * expf(m2 - mm));
    m = mm;
  }
  if (lane == 0) stats[row] = make_float2(m, l > 0.f ? 1.f / l : 0.f);
}

// ---------------------------------------------------------------- probe pass 2
template <int D>
__global__ void __launch_bounds__(128) probe_f32_scores(const float *__restrict__ q, const int32_t *__restrict__ qpos,
                                                        int P, const float *__restrict__ k,
                                                        const int32_t *__restrict__ kpos, int64_t Nc, int Hq,
                                                        int Hkv, float scale, const float2 *__restrict__ stats,
                                                        float *__restrict__ group, float *__restrict__ scores) {
  const int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (j >= Nc) return;
  const int G = Hq / Hkv;
  const int32_t pj = kpos[j];
  float total = 0.f;
  for (int g = 0; g < Hkv; ++g) {
    __align__(16) float kr[D];
#pragma unroll
    for (int t = 0; t < D; t += 4)
      *reinterpret_cast<float4 *>(kr + t) = __ldg(reinterpret_cast<const float4 *>(k + (j * Hkv + g) * D + t));
    float acc = 0.f;
    for (int hh = 0; hh < G; ++hh) {
      const int h = g * G + hh;
      for (int p = 0; p < P; ++p) {
        if (pj > qpos[p]) continue;
        const float x = dot_row<D>(kr, q + (static_cast<int64_t>(p) * Hq + h) * D) * scale;
        const float2 st = stats[h * P + p];
        acc += expf(x - st.x) * st.y;
      }
    }
    if (group) group[g * Nc + j] = acc;
    total += acc;
  }
  scores[j] = total;
}

spts_status launch_probe_f32(const float *q, const int32_t *qpos, int P, const float *k, const int32_t *kpos,
                             int64_t Nc, int Hq, int Hkv, int d, float scale, float *scores, float *group,
                             float *row_stats, cudaStream_t s) {
  float2 *stats = reinterpret_cast<float2 *>(row_stats);
  const unsigned b1 = static_cast<unsigned>((Hq * P + 7) / 8);
  const unsigned b2 = static_cast<unsigned>((Nc + 127) / 128);
  if (d == 64) {
    probe_f32_stats<64><<<b1, 256, 0, s>>>(q, qpos, P, k, kpos, Nc, Hq, Hkv, scale, stats);
    note_launch();
    probe_f32_scores<64><<<b2, 128, 0, s>>>(q, qpos, P, k, kpos, Nc, Hq, Hkv, scale, stats, group, scores);
    note_launch();
  } else {
    probe_f32_stats<128><<<b1, 256, 0, s>>>(q, qpos, P, k, kpos, Nc, Hq, Hkv, scale, stats);
    note_launch();
    probe_f32_scores<128><<<b2, 128, 0, s>>>(q, qpos, P, k, kpos, Nc, Hq, Hkv, scale, stats, group, scores);
    note_launch();
  }
  SPTS_CUDA_TRY(cudaGetLastError());
  return SPTS_OK;
}

// ---------------------------------------------------------------- attention
template <int D>
__global__ void __launch_bounds__(256) attention_f32_kernel(const float *__restrict__ q,
                                                            const int32_t *__restrict__ qpos, int64_t m,
                                                            const float *__restrict__ k,
                                                            const float *__restrict__ v,
                                                            const int32_t *__restrict__ kpos, int64_t Nc, int Hq,
                                                            int Hkv, float scale, float *__restrict__ o) {
  constexpr int C = D / 32;  // output columns per lane
  __shared__ __align__(16) float qs[8][D];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t task = static_cast<int64_t>(blockIdx.x) * 8 + w;  // task = i * Hq + h
  const bool live = task < m * Hq;
  const int64_t i = live ? task / Hq : 0;
  const int h = live ? static_cast<int>(task % Hq) : 0;
  const int g = h / (Hq / Hkv);
  for (int t = lane; t < D; t += 32) qs[w][t] = live ? q[(i * Hq + h) * D + t] * scale : 0.f;
  __syncwarp();
  if (!live) return;
  const int32_t lim = qpos[i];
  float mrow = -INFINITY, l = 0.f, acc[C];
#pragma unroll
  for (int c = 0; c < C; ++c) acc[c] = 0.f;
  for (int64_t j0 = 0; j0 < Nc; j0 += 32) {
    const int64_t j = j0 + lane;
    const bool vis = j < Nc && kpos[j] <= lim;
    const float x = vis ? dot_row<D>(qs[w], k + (j * Hkv + g) * D) : -INFINITY;
    float cm = x;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, off));
    if (cm == -INFINITY) {
      if (kpos[min(j0, Nc - 1)] > lim) break;  // keys ascend: nothing visible later
      continue;
    }
    const float mnew = fmaxf(mrow, cm);
    const float corr = (mrow == -INFINITY) ? 0.f : expf(mrow - mnew);
    const float pj = vis ? expf(x - mnew) : 0.f;
    float ps = pj;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
    l = l * corr + ps;
#pragma unroll
    for (int c = 0; c < C; ++c) acc[c] *= corr;
    const int64_t jmax = min(static_cast<int64_t>(32), Nc - j0);
    for (int t = 0; t < jmax; ++t) {
      const float pt = __shfl_sync(0xffffffffu, pj, t);
      if (pt == 0.f) continue;
      const float *vr = v + ((j0 + t) * Hkv + g) * D;
#pragma unroll
      for (int c = 0; c < C; ++c) acc[c] = fmaf(pt, __ldg(vr + lane + 32 * c), acc[c]);
    }
    mrow = mnew;
  }
  const float inv = l > 0.f ? 1.f / l : 0.f;
  float *orow = o + (i * Hq + h) * D;
#pragma unroll
  for (int c = 0; c < C; ++c) orow[lane + 32 * c] = acc[c] * inv;
}

spts_status launch_attention_f32(const float *q, const int32_t *qpos, int64_t m, const float *k, const float *v,
                                 const int32_t *kpos, int64_t Nc, int Hq, int Hkv, int d, float scale, float *o,
                                 cudaStream_t s) {
  if (m == 0) return SPTS_OK;
  const unsigned blocks = static_cast<unsigned>((m * Hq + 7) / 8);
  if (d == 64)
    attention_f32_kernel<64><<<blocks, 256, 0, s>>>(q, qpos, m, k, v, kpos, Nc, Hq, Hkv, scale, o);
  else
    attention_f32_kernel<128><<<blocks, 256, 0, s>>>(q, qpos, m, k, v, kpos, Nc, Hq, Hkv, scale, o);
  note_launch();
  SPTS_CUDA_TRY(cudaGetLastError());
  return SPTS_OK;
}

}  // namespace spts
