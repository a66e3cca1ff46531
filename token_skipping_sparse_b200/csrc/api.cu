// api.cu -- the extern "C" entry points of libspts: host-side validation,
// workspace carving and dispatch to the kernels.  See include/spts.h for the
// contract of every call.
#include <cmath>

#include "host.hpp"
#include "rowops.cuh"

using namespace spts;

namespace {

inline cudaStream_t cs(spts_stream s) { return reinterpret_cast<cudaStream_t>(s); }

spts_status check_attn(const spts_attn_desc *a, const char *who) {
  SPTS_REQUIRE(a != nullptr, SPTS_ERR_INVALID, "%s: attention descriptor is NULL", who);
  SPTS_REQUIRE(a->Hq > 0 && a->Hkv > 0 && a->Hq % a->Hkv == 0, SPTS_ERR_SHAPE,
               "%s: need Hq, Hkv > 0 and Hq %% Hkv == 0 (Hq=%d Hkv=%d)", who, a->Hq, a->Hkv);
  SPTS_REQUIRE(a->dtype == SPTS_F32 || a->dtype == SPTS_BF16, SPTS_ERR_INVALID, "%s: unknown dtype", who);
  SPTS_REQUIRE(a->d == 64 || a->d == 128, SPTS_ERR_SHAPE, "%s: head dim must be 64 or 128 (d=%d)", who, a->d);
  if (a->dtype == SPTS_BF16) {
    SPTS_REQUIRE(a->d == 128, SPTS_ERR_UNSUPPORTED, "%s: bf16 path needs d = 128 (d=%d)", who, a->d);
    const int G = a->Hq / a->Hkv;
    SPTS_REQUIRE(G == 1 || G == 2 || G == 4 || G == 8, SPTS_ERR_UNSUPPORTED,
                 "%s: bf16 path needs Hq/Hkv in {1,2,4,8} (got %d)", who, G);
  }
  return SPTS_OK;
}

inline float attn_scale(const spts_attn_desc *a) {
  return a->scale > 0.f ? a->scale : 1.0f / std::sqrt(static_cast<float>(a->d));
}

}  // namespace

extern "C" {

// ------------------------------------------------------------------ probe
size_t spts_probe_scores_workspace(const spts_attn_desc *a, int P, int64_t Nc) {
  if (a == nullptr || P <= 0 || Nc <= 0) return kStatusBytes;
  size_t b = kStatusBytes;
  b += Carver::round(static_cast<size_t>(a->Hkv) * Nc * sizeof(float));  // group scores
  if (a->dtype == SPTS_F32)
    b += Carver::round(static_cast<size_t>(a->Hq) * P * sizeof(float) * 2);
  else
    b += Carver::round(probe_bf16_stats_bytes(P, a->Hq, Nc));
  return b;
}

spts_status spts_probe_scores(const spts_attn_desc *a, const void *q_probe, const int32_t *probe_pos, int P,
                              const void *k, const int32_t *key_pos, int64_t Nc, float *scores,
                              float *group_scores, void *ws, size_t ws_bytes, spts_stream stream) {
  const char *who = "spts_probe_scores";
  SPTS_TRY(check_attn(a, who));
  SPTS_REQUIRE(q_probe && probe_pos && k && key_pos && scores, SPTS_ERR_INVALID, "%s: NULL argument", who);
  SPTS_REQUIRE(P >= 1 && P <= 128 && Nc >= 1 && P <= Nc && Nc < (int64_t(1) << 31), SPTS_ERR_SHAPE,
               "%s: need 1 <= P <= 128, P <= Nc < 2^31 (P=%d Nc=%lld)", who, P, static_cast<long long>(Nc));
  SPTS_REQUIRE(aligned(q_probe, 16) && aligned(k, 16) && aligned(scores, 4) && aligned(probe_pos, 4) &&
                   aligned(key_pos, 4) && (!group_scores || aligned(group_scores, 4)),
               SPTS_ERR_INVALID, "%s: misaligned pointer", who);
  SPTS_TRY(check_ws(ws, ws_bytes, spts_probe_scores_workspace(a, P, Nc), who));
  Carver cv(ws, ws_bytes);
  float *group = static_cast<float *>(cv.take(static_cast<size_t>(a->Hkv) * Nc * sizeof(float)));
  if (group_scores) group = group_scores;
  const float sc = attn_scale(a);
  if (a->dtype == SPTS_F32) {
    float *stats = static_cast<float *>(cv.take(static_cast<size_t>(a->Hq) * P * sizeof(float) * 2));
    return launch_probe_f32(static_cast<const float *>(q_probe), probe_pos, P, static_cast<const float *>(k),
                            key_pos, Nc, a->Hq, a->Hkv, a->d, sc, scores, group, stats, cs(stream));
  }
  float *stats = static_cast<float *>(cv.take(probe_bf16_stats_bytes(P, a->Hq, Nc)));
  SPTS_TRY(launch_probe_bf16(q_probe, probe_pos, P, k, key_pos, Nc, a->Hq, a->Hkv, sc, group, stats,
                             cv.status(), cs(stream)));
  return launch_sum_groups(group, a->Hkv, Nc, scores, cs(stream));
}

// ------------------------------------------------------------------ LTP
size_t spts_ltp_scores_workspace(int64_t, int, int r, int) { return kStatusBytes + Carver::round(ltp_gram_bytes(r)); }

spts_status spts_ltp_scores(spts_dtype dt, const void *x, int64_t Nc, int D, const void *A, int r, const void *B,
                            int Dout, float *scores, void *ws, size_t ws_bytes, spts_stream stream) {
  const char *who = "spts_ltp_scores";
  SPTS_REQUIRE(dt == SPTS_BF16, SPTS_ERR_UNSUPPORTED, "%s: only bf16 is supported", who);
  SPTS_REQUIRE(Nc == 0 || (x && scores), SPTS_ERR_INVALID, "%s: NULL argument", who);
  SPTS_REQUIRE(A && B, SPTS_ERR_INVALID, "%s: NULL weights", who);
  SPTS_REQUIRE(Nc >= 0 && D > 0 && D % 64 == 0 && r >= 64 && r <= 256 && r % 64 == 0 && Dout > 0 &&
                   Dout % 256 == 0,
               SPTS_ERR_SHAPE, "%s: need D%%64==0, r in {64..256} step 64, Dout%%256==0 (D=%d r=%d Dout=%d)",
               who, D, r, Dout);
  SPTS_REQUIRE(aligned(x, 16) && aligned(A, 16) && aligned(B, 16) && aligned(scores, 4), SPTS_ERR_INVALID,
               "%s: misaligned pointer", who);
  SPTS_TRY(check_ws(ws, ws_bytes, spts_ltp_scores_workspace(Nc, D, r, Dout), who));
  if (Nc == 0) return SPTS_OK;
  Carver cv(ws, ws_bytes);
  void *gram = cv.take(ltp_gram_bytes(r));
  return launch_ltp_bf16(x, Nc, D, A, r, B, Dout, scores, cv.status(), cs(stream), 0, gram);
}

size_t spts_ltp_topm_scores_workspace(int64_t, int, int, int) { return kStatusBytes; }

spts_status spts_ltp_topm_scores(spts_dtype dt, const void *x, int64_t Nc, int D, const void *A, int r,
                                 const void *B, int Dout, int top_m, float *scores, void *ws, size_t ws_bytes,
                                 spts_stream stream) {
  const char *who = "spts_ltp_topm_scores";
  SPTS_REQUIRE(dt == SPTS_BF16, SPTS_ERR_UNSUPPORTED, "%s: only bf16 is supported", who);
  SPTS_REQUIRE(Nc == 0 || (x && scores), SPTS_ERR_INVALID, "%s: NULL argument", who);
  SPTS_REQUIRE(A && B, SPTS_ERR_INVALID, "%s: NULL weights", who);
  SPTS_REQUIRE(Nc >= 0 && D > 0 && D % 64 == 0 && r >= 64 && r <= 256 && r % 64 == 0 &&
                   (Dout == 256 || Dout == 512) && top_m >= 1 && top_m <= Dout,
               SPTS_ERR_SHAPE,
               "%s: need D%%64==0, r in {64..256} step 64, Dout in {256, 512}, 1 <= top_m <= Dout (D=%d r=%d "
               "Dout=%d top_m=%d)",
               who, D, r, Dout, top_m);
  SPTS_REQUIRE(aligned(x, 16) && aligned(A, 16) && aligned(B, 16) && aligned(scores, 4), SPTS_ERR_INVALID,
               "%s: misaligned pointer", who);
  SPTS_TRY(check_ws(ws, ws_bytes, spts_ltp_topm_scores_workspace(Nc, D, r, Dout), who));
  if (Nc == 0) return SPTS_OK;
  return launch_ltp_bf16(x, Nc, D, A, r, B, Dout, scores, static_cast<uint32_t *>(ws), cs(stream), top_m, nullptr);
}

// ------------------------------------------------------------------ select
size_t spts_select_topk_workspace(int64_t Nc) {
  return kStatusBytes + Carver::round(topk_scratch_bytes(Nc));
}

spts_status spts_select_topk(const float *s_a, const float *s_b, spts_fuse mode, float w_a, float w_b,
                             int64_t Nc, int64_t k, int64_t force_tail, int32_t *idx_out, float *fused_out,
                             float *kth_score_out, void *ws, size_t ws_bytes, spts_stream stream) {
  const char *who = "spts_select_topk";
  SPTS_REQUIRE(mode == SPTS_FUSE_NONE || mode == SPTS_FUSE_MAXNORM_ADD || mode == SPTS_FUSE_MULTIPLY ||
                   mode == SPTS_FUSE_STD_ADD,
               SPTS_ERR_INVALID, "%s: unknown fusion mode %d", who, static_cast<int>(mode));
  SPTS_REQUIRE(Nc == 0 || (s_a && idx_out && (mode == SPTS_FUSE_NONE || s_b)), SPTS_ERR_INVALID, "%s: NULL argument", who);
  SPTS_REQUIRE(0 <= force_tail && force_tail <= k && k <= Nc && Nc < (int64_t(1) << 31), SPTS_ERR_SHAPE,
               "%s: need 0 <= force_tail <= k <= Nc < 2^31 (tail=%lld k=%lld Nc=%lld)", who,
               static_cast<long long>(force_tail), static_cast<long long>(k), static_cast<long long>(Nc));
  SPTS_REQUIRE(std::isfinite(w_a) && std::isfinite(w_b), SPTS_ERR_INVALID, "%s: non-finite weight", who);
  SPTS_REQUIRE(aligned(s_a, 4) && (!s_b || aligned(s_b, 4)) && aligned(idx_out, 4), SPTS_ERR_INVALID,
               "%s: misaligned pointer", who);
  SPTS_TRY(check_ws(ws, ws_bytes, spts_select_topk_workspace(Nc), who));
  if (Nc == 0) return SPTS_OK;
  Carver cv(ws, ws_bytes);
  void *scratch = cv.take(topk_scratch_bytes(Nc));
  return launch_select_topk(s_a, s_b, mode, w_a, w_b, Nc, k, force_tail, idx_out, fused_out, kth_score_out,
                            cv.status(), scratch, cs(stream));
}

size_t spts_select_sequential_workspace(int64_t Nc) {
  return kStatusBytes + Carver::round(select_sequential_scratch_bytes(Nc));
}

spts_status spts_select_sequential(const float *s_a, const float *s_b, int64_t Nc, int64_t k_pool, int64_t k,
                                   int64_t force_tail, int32_t *idx_out, void *ws, size_t ws_bytes,
                                   spts_stream stream) {
  const char *who = "spts_select_sequential";
  SPTS_REQUIRE(Nc == 0 || (s_a && s_b && idx_out), SPTS_ERR_INVALID, "%s: NULL argument", who);
  SPTS_REQUIRE(0 <= force_tail && force_tail <= k && k <= k_pool && k_pool <= Nc && Nc < (int64_t(1) << 31),
               SPTS_ERR_SHAPE, "%s: need 0 <= force_tail <= k <= k_pool <= Nc < 2^31 (tail=%lld k=%lld pool=%lld "
               "Nc=%lld)", who, static_cast<long long>(force_tail), static_cast<long long>(k),
               static_cast<long long>(k_pool), static_cast<long long>(Nc));
  SPTS_REQUIRE(aligned(s_a, 4) && aligned(s_b, 4) && aligned(idx_out, 4), SPTS_ERR_INVALID,
               "%s: misaligned pointer", who);
  SPTS_TRY(check_ws(ws, ws_bytes, spts_select_sequential_workspace(Nc), who));
  if (Nc == 0 || k == 0) return SPTS_OK;
  Carver cv(ws, ws_bytes);
  void *scratch = cv.take(select_sequential_scratch_bytes(Nc));
  return launch_select_sequential(s_a, s_b, Nc, k_pool, k, force_tail, idx_out, scratch, cv.status(), cs(stream));
}

// ------------------------------------------------------------------ attention
size_t spts_reduced_attention_workspace(const spts_attn_desc *, int64_t, int64_t) { return kStatusBytes; }

spts_status spts_reduced_attention(const spts_attn_desc *a, const void *q_sel, const int32_t *q_pos, int64_t k,
                                   const void *kk, const void *v, const int32_t *key_pos, int64_t Nc, void *o_sel,
                                   void *ws, size_t ws_bytes, spts_stream stream) {
  const char *who = "spts_reduced_attention";
  SPTS_TRY(check_attn(a, who));
  SPTS_REQUIRE(q_sel && q_pos && kk && v && key_pos && o_sel, SPTS_ERR_INVALID, "%s: NULL argument", who);
  SPTS_REQUIRE(k >= 0 && Nc >= 1 && Nc < (int64_t(1) << 31) && k < (int64_t(1) << 31), SPTS_ERR_SHAPE,
               "%s: bad sizes (k=%lld Nc=%lld)", who, static_cast<long long>(k), static_cast<long long>(Nc));
  SPTS_REQUIRE(aligned(q_sel, 16) && aligned(kk, 16) && aligned(v, 16) && aligned(o_sel, 16) &&
                   aligned(q_pos, 4) && aligned(key_pos, 4),
               SPTS_ERR_INVALID, "%s: misaligned pointer", who);
  SPTS_REQUIRE(o_sel != q_sel, SPTS_ERR_INVALID, "%s: o_sel must not alias q_sel", who);
  SPTS_TRY(check_ws(ws, ws_bytes, spts_reduced_attention_workspace(a, k, Nc), who));
  if (k == 0) return SPTS_OK;
  const float sc = attn_scale(a);
  if (a->dtype == SPTS_F32)
    return launch_attention_f32(static_cast<const float *>(q_sel), q_pos, k, static_cast<const float *>(kk),
                                static_cast<const float *>(v), key_pos, Nc, a->Hq, a->Hkv, a->d, sc,
                                static_cast<float *>(o_sel), cs(stream));
  return launch_attention_bf16(q_sel, q_pos, k, kk, v, key_pos, Nc, a->Hq, a->Hkv, sc, o_sel,
                               static_cast<uint32_t *>(ws), cs(stream));
}

// ------------------------------------------------------------------ FFN
size_t spts_reduced_ffn_workspace(int64_t k, int D, int F) {
  size_t b = kStatusBytes;
  b += Carver::round(static_cast<size_t>(k) * D * 2);  // gathered, normalized rows (bf16)
  b += Carver::round(static_cast<size_t>(k) * F * 2);  // SwiGLU activation (bf16)
  return b;
}

spts_status spts_reduced_ffn(spts_dtype dt, float *h, int64_t Nc, int D, const int32_t *idx, int64_t k,
                             const void *norm_w, float eps, const void *w_gate, const void *w_up,
                             const void *w_down, int F, void *ws, size_t ws_bytes, spts_stream stream) {
  const char *who = "spts_reduced_ffn";
  SPTS_REQUIRE(dt == SPTS_BF16, SPTS_ERR_UNSUPPORTED, "%s: only bf16 weights are supported", who);
  SPTS_REQUIRE((k == 0 || (h && idx)) && w_gate && w_up && w_down, SPTS_ERR_INVALID, "%s: NULL argument", who);
  SPTS_REQUIRE(k >= 0 && k <= Nc && D > 0 && D % 256 == 0 && F > 0 && F % 128 == 0, SPTS_ERR_SHAPE,
               "%s: need k <= Nc, D %% 256 == 0, F %% 128 == 0 (k=%lld Nc=%lld D=%d F=%d)", who,
               static_cast<long long>(k), static_cast<long long>(Nc), D, F);
  SPTS_REQUIRE(aligned(h, 16) && aligned(w_gate, 16) && aligned(w_up, 16) && aligned(w_down, 16) &&
                   aligned(idx, 4) && (!norm_w || aligned(norm_w, 16)),
               SPTS_ERR_INVALID, "%s: misaligned pointer", who);
  SPTS_REQUIRE(eps >= 0.f, SPTS_ERR_INVALID, "%s: eps must be >= 0", who);
  SPTS_TRY(check_ws(ws, ws_bytes, spts_reduced_ffn_workspace(k, D, F), who));
  if (k == 0) return SPTS_OK;
  Carver cv(ws, ws_bytes);
  void *x = cv.take(static_cast<size_t>(k) * D * 2);
  void *act = cv.take(static_cast<size_t>(k) * F * 2);
  cudaStream_t s = cs(stream);
  SPTS_TRY(launch_rmsnorm_rows(h, idx, k, D, norm_w, eps, x, s));
  GemmArgs g1{x, k, D, w_gate, w_up, F, SPTS_EPI_SWIGLU, act, nullptr, nullptr, 0.0, cv.status()};
  SPTS_TRY(launch_gemm(g1, s));
  GemmArgs g2{act, k, F, w_down, nullptr, D, SPTS_EPI_SCATTER_ADD, h, idx, nullptr, 0.0, cv.status()};
  return launch_gemm(g2, s);
}

// ------------------------------------------------------------------ MSDP prune
size_t spts_stage_prune_workspace(int64_t Nc) {
  return kStatusBytes + Carver::round(Nc * sizeof(int32_t)) + Carver::round(topk_scratch_bytes(Nc));
}

spts_status spts_stage_prune(const float *scores, int64_t Nc, int64_t k_keep, int64_t force_tail,
                             const float *h_in, const int32_t *pos_in, int D, float *h_out, int32_t *pos_out,
                             int32_t *kept_idx, void *ws, size_t ws_bytes, spts_stream stream) {
  const char *who = "spts_stage_prune";
  SPTS_REQUIRE(scores && h_in && pos_in && h_out && pos_out, SPTS_ERR_INVALID, "%s: NULL argument", who);
  SPTS_REQUIRE(0 <= force_tail && force_tail <= k_keep && k_keep <= Nc && Nc < (int64_t(1) << 31) && D > 0 &&
                   D % 4 == 0,
               SPTS_ERR_SHAPE, "%s: need 0 <= force_tail <= k_keep <= Nc and D %% 4 == 0", who);
  SPTS_REQUIRE(aligned(h_in, 16) && aligned(h_out, 16) && aligned(scores, 4) && aligned(pos_in, 4) &&
                   aligned(pos_out, 4),
               SPTS_ERR_INVALID, "%s: misaligned pointer", who);
  const char *hi = reinterpret_cast<const char *>(h_in), *ho = reinterpret_cast<const char *>(h_out);
  const size_t hb = static_cast<size_t>(Nc) * D * 4, ob = static_cast<size_t>(k_keep) * D * 4;
  SPTS_REQUIRE(ho + ob <= hi || hi + hb <= ho, SPTS_ERR_INVALID, "%s: h_out overlaps h_in", who);
  SPTS_TRY(check_ws(ws, ws_bytes, spts_stage_prune_workspace(Nc), who));
  if (k_keep == 0) return SPTS_OK;
  Carver cv(ws, ws_bytes);
  int32_t *kept = static_cast<int32_t *>(cv.take(Nc * sizeof(int32_t)));
  if (kept_idx) kept = kept_idx;
  void *scratch = cv.take(topk_scratch_bytes(Nc));
  cudaStream_t s = cs(stream);
  SPTS_TRY(launch_select_topk(scores, nullptr, SPTS_FUSE_NONE, 0.f, 0.f, Nc, k_keep, force_tail, kept, nullptr,
                              nullptr, cv.status(), scratch, s));
  return launch_gather_rows(h_in, Nc, kept, k_keep, static_cast<int64_t>(D) * 4, h_out, pos_in, pos_out,
                            cv.status(), s);
}

// ------------------------------------------------------------------ supporting calls
spts_status spts_rmsnorm_rows(const float *x, const int32_t *rows, int64_t m, int D, const void *w, float eps,
                              void *y, spts_stream stream) {
  const char *who = "spts_rmsnorm_rows";
  SPTS_REQUIRE(m == 0 || (x && y), SPTS_ERR_INVALID, "%s: NULL argument", who);
  SPTS_REQUIRE(m >= 0 && D > 0 && D % 8 == 0, SPTS_ERR_SHAPE, "%s: need D %% 8 == 0", who);
  SPTS_REQUIRE(aligned(x, 16) && aligned(y, 16) && (!w || aligned(w, 16)) && (!rows || aligned(rows, 4)),
               SPTS_ERR_INVALID, "%s: misaligned pointer", who);
  return launch_rmsnorm_rows(x, rows, m, D, w, eps, y, cs(stream));
}

spts_status spts_rope(void *x, int64_t m, int H, int d, const int32_t *pos, double theta, spts_stream stream) {
  const char *who = "spts_rope";
  SPTS_REQUIRE(m == 0 || (x && pos), SPTS_ERR_INVALID, "%s: NULL argument", who);
  SPTS_REQUIRE(m >= 0 && H > 0 && d > 0 && d % 2 == 0 && d <= 256 && theta > 0, SPTS_ERR_SHAPE,
               "%s: need even d <= 256 and theta > 0", who);
  return launch_rope(x, m, H, d, pos, theta, cs(stream));
}

spts_status spts_gather_rows(const void *src, int64_t n_src, const int32_t *rows, int64_t m, int64_t row_bytes,
                             void *dst, void *ws, spts_stream stream) {
  const char *who = "spts_gather_rows";
  SPTS_REQUIRE(m == 0 || (src && rows && dst), SPTS_ERR_INVALID, "%s: NULL argument", who);
  SPTS_REQUIRE(m >= 0 && n_src >= 0 && row_bytes > 0 && row_bytes % 16 == 0, SPTS_ERR_SHAPE,
               "%s: row_bytes must be a positive multiple of 16", who);
  SPTS_REQUIRE(aligned(src, 16) && aligned(dst, 16) && aligned(rows, 4), SPTS_ERR_INVALID,
               "%s: misaligned pointer", who);
  return launch_gather_rows(src, n_src, rows, m, row_bytes, dst, nullptr, nullptr, static_cast<uint32_t *>(ws),
                            cs(stream));
}

size_t spts_linear_workspace(void) { return kStatusBytes; }

spts_status spts_linear(const void *A, int64_t M, int K, const void *W, const void *W2, int N, spts_epilogue epi,
                        void *out, const int32_t *rows, const int32_t *row_pos, double theta, void *ws,
                        size_t ws_bytes, spts_stream stream) {
  const char *who = "spts_linear";
  SPTS_REQUIRE(W && (M == 0 || (A && out)), SPTS_ERR_INVALID, "%s: NULL argument", who);
  SPTS_REQUIRE(epi >= SPTS_EPI_STORE && epi <= SPTS_EPI_SCATTER_ADD, SPTS_ERR_INVALID, "%s: bad epilogue", who);
  SPTS_REQUIRE(M >= 0 && M < (int64_t(1) << 31) && K > 0 && K % 64 == 0 && N > 0, SPTS_ERR_SHAPE,
               "%s: need K %% 64 == 0 (K=%d)", who, K);
  if (epi == SPTS_EPI_SWIGLU) {
    SPTS_REQUIRE(W2 != nullptr, SPTS_ERR_INVALID, "%s: SWIGLU needs W2 (W_up)", who);
    SPTS_REQUIRE(N % 128 == 0, SPTS_ERR_SHAPE, "%s: SWIGLU needs N %% 128 == 0", who);
  } else {
    SPTS_REQUIRE(N % 256 == 0, SPTS_ERR_SHAPE, "%s: need N %% 256 == 0 (N=%d)", who, N);
  }
  if (epi == SPTS_EPI_ROPE) SPTS_REQUIRE(row_pos != nullptr && theta > 0, SPTS_ERR_INVALID, "%s: ROPE needs row_pos", who);
  if (epi == SPTS_EPI_SCATTER_ADD) SPTS_REQUIRE(rows != nullptr, SPTS_ERR_INVALID, "%s: SCATTER_ADD needs rows", who);
  SPTS_REQUIRE(aligned(A, 16) && aligned(W, 16) && (!W2 || aligned(W2, 16)) && aligned(out, 16), SPTS_ERR_INVALID,
               "%s: misaligned pointer", who);
  SPTS_TRY(check_ws(ws, ws_bytes, spts_linear_workspace(), who));
  GemmArgs g{A, M, K, W, W2, N, static_cast<int>(epi), out, rows, row_pos, theta, static_cast<uint32_t *>(ws)};
  return launch_gemm(g, cs(stream));
}

spts_status spts_inject_salience(void *k, int64_t Nc, const void *q_probe, int P, int Hq, int Hkv, int d,
                                 const int32_t *rows, int64_t n_rows, float shift, spts_stream stream) {
  const char *who = "spts_inject_salience";
  SPTS_REQUIRE(k && q_probe && (rows || n_rows == 0), SPTS_ERR_INVALID, "%s: NULL argument", who);
  SPTS_REQUIRE(Hq > 0 && Hkv > 0 && Hq % Hkv == 0 && d > 0 && d <= 1024 && (d & (d - 1)) == 0 && P > 0,
               SPTS_ERR_SHAPE, "%s: bad geometry", who);
  return launch_inject_salience(k, Nc, q_probe, P, Hq, Hkv, d, rows, n_rows, shift, nullptr, cs(stream));
}

spts_status spts_debug_exp2_poly(const float *x, int64_t n, float *y, spts_stream stream) {
  const char *who = "spts_debug_exp2_poly";
  SPTS_REQUIRE(n >= 0, SPTS_ERR_SHAPE, "%s: n < 0", who);
  SPTS_REQUIRE(n == 0 || (x && y), SPTS_ERR_INVALID, "%s: NULL argument", who);
  SPTS_REQUIRE(aligned(x, 4) && aligned(y, 4), SPTS_ERR_INVALID, "%s: misaligned pointer", who);
  return launch_exp2_poly(x, n, y, cs(stream));
}

}  // extern "C"
