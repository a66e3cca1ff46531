// rowops.cuh -- launchers of the row kernels, the top-k / prune kernels, and
// the attention, probe, LTP and GEMM kernels (internal interface between the
// C-ABI layer and the kernels).
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

#include "spts.h"

namespace spts {

struct RopeFreqs {
  double inv_freq[128];  // theta^(-2i/d), i < d/2
  // the same frequencies in turns (inv_freq / 2 pi) as two fp32 parts:
  // turn_hi = fp32(g), turn_lo = fp32(g - turn_hi), about 2^-24 g
  float turn_hi[128], turn_lo[128];
};
void fill_rope_freqs(RopeFreqs *f, int d, double theta);

// cos and sin of pos * inv_freq[i].  The angle is reduced in turns without
// fp64 arithmetic: pos * turn_hi = hi + lo exactly (an FMA two-product; pos
// below 2^24 is exact in fp32), the integer part of hi is dropped exactly
// and pos * turn_lo adds the next 24 bits of the frequency, so the reduced
// angle is within ~1e-7 turns; __sincosf then works on [-pi, pi] where its
// error is ~2^-21.  Positions from 2^24 on take an fp64 reduction.
__device__ __forceinline__ void rope_cos_sin(int32_t pos, const RopeFreqs &f, int i, float *c, float *s) {
  float t;
  if (pos < (1 << 24)) {
    const float pf = static_cast<float>(pos);
    const float hi = pf * f.turn_hi[i];
    const float lo = fmaf(pf, f.turn_hi[i], -hi);
    t = (hi - rintf(hi)) + (lo + pf * f.turn_lo[i]);
  } else {
    const double a = static_cast<double>(pos) * f.inv_freq[i] * 0.15915494309189533576888376337251;
    t = static_cast<float>(a - rint(a));
  }
  __sincosf(t * 6.28318530717958647692f, s, c);
}

// Row i of x (x[rows[i]] with rows) normalised into y[i] (y[rows[i]] when
// scatter).
spts_status launch_rmsnorm_rows(const float *x, const int32_t *rows, int64_t m, int D, const void *w, float eps,
                                void *y, cudaStream_t s, bool scatter = false);
spts_status launch_rope(void *x, int64_t m, int H, int d, const int32_t *pos, double theta, cudaStream_t s);
spts_status launch_gather_rows(const void *src, int64_t n_src, const int32_t *rows, int64_t m, int64_t row_bytes,
                               void *dst, const int32_t *pos_in, int32_t *pos_out, uint32_t *status,
                               cudaStream_t s);
spts_status launch_inject_salience(void *k, int64_t Nc, const void *q_probe, int P, int Hq, int Hkv, int d,
                                   const int32_t *rows, int64_t n_rows, float shift, uint32_t *status,
                                   cudaStream_t s);
spts_status launch_gather_i32(const int32_t *src, const int32_t *idx, int64_t m, int32_t *dst, cudaStream_t s);
// Load the kernels of the row gather / the top-k selection on the current
// device now (CUDA loads a kernel's code lazily, at its first launch or
// attribute query), so that a later launch takes no device memory for code.
spts_status preload_gather_rows();
// bf16 residual boundary: n bf16 -> fp32 (n % 8 == 0); rows[t] of src fp32
// -> bf16 into dst (D % 8 == 0).
spts_status launch_bf16_to_f32(const void *src, int64_t n, float *dst, cudaStream_t s);
spts_status launch_exp2_poly(const float *x, int64_t n, float *y, cudaStream_t s);
spts_status launch_rows_f32_to_bf16(const float *src, const int32_t *rows, int64_t m, int64_t n_rows, int D,
                                    void *dst, uint32_t *status, cudaStream_t s);
spts_status preload_select_topk();
spts_status launch_iota_i32(int32_t *dst, int64_t n, cudaStream_t s);
spts_status launch_sum_groups(const float *group, int G, int64_t n, float *s, cudaStream_t st);

// Top-k selection: radix select + stable compaction, on one CTA, or on the
// grid when `scratch` (topk_scratch_bytes(Nc) bytes) is given and the
// candidate set is large.
size_t topk_scratch_bytes(int64_t Nc);
size_t select_sequential_scratch_bytes(int64_t Nc);
spts_status launch_select_sequential(const float *s_a, const float *s_b, int64_t Nc, int64_t k_pool, int64_t k,
                                     int64_t force_tail, int32_t *idx_out, void *scratch, uint32_t *status,
                                     cudaStream_t s);
spts_status launch_select_topk(const float *s_a, const float *s_b, int mode, float w_a, float w_b, int64_t Nc,
                               int64_t k, int64_t force_tail, int32_t *idx_out, float *fused_out,
                               float *kth_out, uint32_t *status, void *scratch, cudaStream_t s);

// fp32 CUDA-core attention paths.
spts_status launch_probe_f32(const float *q, const int32_t *qpos, int P, const float *k, const int32_t *kpos,
                             int64_t Nc, int Hq, int Hkv, int d, float scale, float *scores, float *group,
                             float *row_stats, cudaStream_t s);
spts_status launch_attention_f32(const float *q, const int32_t *qpos, int64_t m, const float *k, const float *v,
                                 const int32_t *kpos, int64_t Nc, int Hq, int Hkv, int d, float scale, float *o,
                                 cudaStream_t s);

// bf16 tensor-core paths (tcgen05).
struct GemmArgs {
  const void *A;
  int64_t M;
  int K;
  const void *W;
  const void *W2;
  int N;
  int epi;
  void *out;
  const int32_t *rows;
  const int32_t *row_pos;
  double theta;
  uint32_t *status;
};
spts_status launch_gemm(const GemmArgs &g, cudaStream_t s);

spts_status launch_probe_bf16(const void *q, const int32_t *qpos, int P, const void *k, const int32_t *kpos,
                              int64_t Nc, int Hq, int Hkv, float scale, float *group, float *row_stats,
                              uint32_t *status, cudaStream_t s);
size_t probe_bf16_stats_bytes(int P, int Hq, int64_t Nc);

// top_m > 0 (Dout <= 512): score = sum of the top_m largest |y| instead of ||y||_2.
// LTP score; top_m == 0 (the L2 norm) needs ltp_gram_bytes(r) of scratch
// for the Gram matrix in gram_ws, top_m > 0 none.
size_t ltp_gram_bytes(int r);
spts_status launch_ltp_bf16(const void *x, int64_t Nc, int D, const void *A, int r, const void *B, int Dout,
                            float *scores, uint32_t *status, cudaStream_t s, int top_m, void *gram_ws);

spts_status launch_attention_bf16(const void *q, const int32_t *qpos, int64_t m, const void *k, const void *v,
                                  const int32_t *kpos, int64_t Nc, int Hq, int Hkv, float scale, void *o,
                                  uint32_t *status, cudaStream_t s);

}  // namespace spts
