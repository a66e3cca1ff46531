// layer.cu -- one SPTS prefill layer composed from the kernels, in the order
// of Fig. 2: probe (PAP) -> select -> reduced attention -> O projection into
// the selected rows -> LTP score -> fuse + select -> reduced FFN.
#include <cstring>
#include <utility>

#include "host.hpp"
#include "rowops.cuh"

using namespace spts;

namespace {

struct LayerBufs {
  void *xn, *kk, *vv, *qprobe, *xsel, *qsel, *osel, *act;
  float *s, *group, *stats, *c, *f;
  int32_t *idx_a, *idx_f, *qpos;
  void *topk;  // scratch of the grid top-k
  void *ksel;  // K of the active rows (kv_active_only)
  void *gram;  // the LTP proxy's Gram matrix (L2-norm score)
};

// Carves the workspace; with cv.base == nullptr it only measures.
void carve(Carver &cv, const spts_layer_desc *L, int64_t Nc, LayerBufs &b) {
  const int64_t k = L->k;
  const size_t D = L->D, hq = static_cast<size_t>(L->Hq) * L->d, hk = static_cast<size_t>(L->Hkv) * L->d;
  b.xn = cv.take(Nc * D * 2);
  b.kk = cv.take(Nc * hk * 2);
  b.vv = cv.take(Nc * hk * 2);
  b.qprobe = cv.take(static_cast<size_t>(L->P) * hq * 2);
  b.xsel = cv.take(k * D * 2);
  b.qsel = cv.take(k * hq * 2);
  b.osel = cv.take(k * hq * 2);
  b.act = cv.take(static_cast<size_t>(k) * (L->F > 0 ? L->F : 1) * 2);
  b.s = static_cast<float *>(cv.take(Nc * 4));
  b.group = static_cast<float *>(cv.take(static_cast<size_t>(L->Hkv) * Nc * 4));
  b.stats = static_cast<float *>(cv.take(probe_bf16_stats_bytes(L->P, L->Hq, Nc)));
  b.c = static_cast<float *>(cv.take(Nc * 4));
  b.f = static_cast<float *>(cv.take(Nc * 4));
  b.idx_a = static_cast<int32_t *>(cv.take(k * 4));
  b.idx_f = static_cast<int32_t *>(cv.take(k * 4));
  b.qpos = static_cast<int32_t *>(cv.take(k * 4));
  b.topk = cv.take(select_sequential_scratch_bytes(Nc));  // also covers the plain top-k
  b.ksel = cv.take(k * hk * 2);
  b.gram = cv.take(L->F > 0 ? ltp_gram_bytes(L->r) : 1);
}

// A side stream and fork/join events per (host thread, device): the V and
// probe-Q projections run on it while the main stream does the K projection,
// the probe scores, the selection and the gathers, which leave most SMs idle.
struct SideStream {
  cudaStream_t s = nullptr;
  cudaEvent_t fork = nullptr, qprobe_done = nullptr, v_done = nullptr;
};

spts_status side_stream(SideStream **out) {
  static thread_local SideStream per_dev[64];
  int dev = 0;
  SPTS_CUDA_TRY(cudaGetDevice(&dev));
  SPTS_REQUIRE(dev >= 0 && dev < 64, SPTS_ERR_UNSUPPORTED, "spts_layer_forward: device ordinal %d", dev);
  SideStream &ss = per_dev[dev];
  if (ss.s == nullptr) {
    SPTS_CUDA_TRY(cudaStreamCreateWithFlags(&ss.s, cudaStreamNonBlocking));
    SPTS_CUDA_TRY(cudaEventCreateWithFlags(&ss.fork, cudaEventDisableTiming));
    SPTS_CUDA_TRY(cudaEventCreateWithFlags(&ss.qprobe_done, cudaEventDisableTiming));
    SPTS_CUDA_TRY(cudaEventCreateWithFlags(&ss.v_done, cudaEventDisableTiming));
  }
  *out = &ss;
  return SPTS_OK;
}

spts_status check_layer(const spts_layer_desc *L, const spts_layer_weights *W, int64_t Nc) {
  const char *who = "spts_layer_forward";
  SPTS_REQUIRE(L && W, SPTS_ERR_INVALID, "%s: NULL descriptor", who);
  SPTS_REQUIRE(L->d == 128 && L->Hq > 0 && L->Hkv > 0 && L->Hq % L->Hkv == 0, SPTS_ERR_UNSUPPORTED,
               "%s: needs d = 128 and Hq %% Hkv == 0", who);
  const int G = L->Hq / L->Hkv;
  SPTS_REQUIRE(G == 1 || G == 2 || G == 4 || G == 8, SPTS_ERR_UNSUPPORTED, "%s: Hq/Hkv must be 1, 2, 4 or 8", who);
  SPTS_REQUIRE(L->D % 256 == 0 && (L->Hq * L->d) % 256 == 0 && (L->Hkv * L->d) % 256 == 0, SPTS_ERR_SHAPE,
               "%s: D, Hq*d and Hkv*d must be multiples of 256", who);
  SPTS_REQUIRE(L->P >= 1 && L->P <= 128 && L->P <= L->k && L->k <= Nc && Nc < (int64_t(1) << 31), SPTS_ERR_SHAPE,
               "%s: need 1 <= P <= 128, P <= k <= Nc", who);
  SPTS_REQUIRE(W->w_q && W->w_k && W->w_v && W->w_o, SPTS_ERR_INVALID, "%s: attention weights missing", who);
  if (L->F > 0) {
    SPTS_REQUIRE(L->F % 128 == 0 && L->r >= 64 && L->r <= 256 && L->r % 64 == 0, SPTS_ERR_SHAPE,
                 "%s: need F %% 128 == 0 and r in {64,...,256} step 64", who);
    SPTS_REQUIRE(W->w_gate && W->w_up && W->w_down && W->ltp_a && W->ltp_b, SPTS_ERR_INVALID,
                 "%s: FFN / LTP weights missing", who);
    SPTS_REQUIRE(L->fuse >= SPTS_FUSE_NONE && L->fuse <= SPTS_FUSE_SEQUENTIAL, SPTS_ERR_INVALID, "%s: bad fusion",
                 who);
    SPTS_REQUIRE(L->fuse != SPTS_FUSE_SEQUENTIAL || L->seq_pool == 0 || (L->seq_pool >= L->k && L->seq_pool <= Nc),
                 SPTS_ERR_SHAPE, "%s: seq_pool must be 0 or in [k, Nc]", who);
    SPTS_REQUIRE(L->ltp_dout == 0 || (L->ltp_dout > 0 && L->ltp_dout % 256 == 0), SPTS_ERR_SHAPE,
                 "%s: ltp_dout must be 0 (= D) or a multiple of 256", who);
    const int dlow = L->ltp_dout > 0 ? L->ltp_dout : L->D;
    SPTS_REQUIRE(L->ltp_top_m == 0 || ((dlow == 256 || dlow == 512) && L->ltp_top_m >= 1 && L->ltp_top_m <= dlow),
                 SPTS_ERR_SHAPE, "%s: ltp_top_m needs D_low in {256, 512} and 1 <= ltp_top_m <= D_low", who);
  }
  SPTS_REQUIRE(L->kv_active_only == 0 || L->kv_active_only == 1, SPTS_ERR_INVALID, "%s: kv_active_only is 0 or 1",
               who);
  SPTS_REQUIRE(L->n_salient == 0 || L->salient_rows != nullptr, SPTS_ERR_INVALID, "%s: salient rows NULL", who);
  return SPTS_OK;
}

// keep 1.0 (k == Nc) with no score outputs asked for and no planted salience:
// every selection is the identity, so the layer is the dense Llama layer --
// no probe, no LTP, no selections, no gathers.
spts_status dense_layer(const spts_layer_desc *L, const spts_layer_weights *W, float *h, const int32_t *pos,
                        int64_t Nc, const spts_layer_outputs &o, const LayerBufs &b, uint32_t *st, cudaStream_t s) {
  const int D = L->D, hq = L->Hq * L->d, hk = L->Hkv * L->d;
  const float scale = 1.0f / sqrtf(static_cast<float>(L->d));
  void *osel = o.o_sel ? o.o_sel : b.osel;
  auto mark = [&](int i) -> spts_status {
    if (o.stage_events != nullptr && o.stage_events[i] != nullptr)
      SPTS_CUDA_TRY(cudaEventRecord(static_cast<cudaEvent_t>(o.stage_events[i]), s));
    return SPTS_OK;
  };
  SPTS_TRY(mark(0));
  SPTS_TRY(launch_rmsnorm_rows(h, nullptr, Nc, D, W->norm_attn, L->eps, b.xn, s));
  SPTS_TRY(mark(1));
  GemmArgs gk{b.xn, Nc, D, W->w_k, nullptr, hk, SPTS_EPI_ROPE, b.kk, nullptr, pos, L->theta, st};
  SPTS_TRY(launch_gemm(gk, s));
  SPTS_TRY(mark(2));
  GemmArgs gv{b.xn, Nc, D, W->w_v, nullptr, hk, SPTS_EPI_STORE, b.vv, nullptr, nullptr, 0.0, st};
  SPTS_TRY(launch_gemm(gv, s));
  for (int i = 3; i <= 7; ++i) SPTS_TRY(mark(i));
  GemmArgs gq{b.xn, Nc, D, W->w_q, nullptr, hq, SPTS_EPI_ROPE, b.qsel, nullptr, pos, L->theta, st};
  SPTS_TRY(launch_gemm(gq, s));
  SPTS_TRY(mark(8));
  SPTS_TRY(launch_attention_bf16(b.qsel, pos, Nc, b.kk, b.vv, pos, Nc, L->Hq, L->Hkv, scale, osel, st, s));
  SPTS_TRY(mark(9));
  SPTS_TRY(launch_iota_i32(b.idx_a, Nc, s));
  GemmArgs go{osel, Nc, hq, W->w_o, nullptr, D, SPTS_EPI_SCATTER_ADD, h, b.idx_a, nullptr, 0.0, st};
  SPTS_TRY(launch_gemm(go, s));
  if (o.h_attn) SPTS_CUDA_TRY(cudaMemcpyAsync(o.h_attn, h, static_cast<size_t>(Nc) * D * 4, cudaMemcpyDeviceToDevice, s));
  SPTS_TRY(mark(10));
  if (L->F <= 0) {
    for (int i = 11; i < SPTS_LAYER_STAGE_EVENTS; ++i) SPTS_TRY(mark(i));
    return SPTS_OK;
  }
  SPTS_TRY(launch_rmsnorm_rows(h, nullptr, Nc, D, W->norm_ffn, L->eps, b.xn, s));
  for (int i = 11; i <= 13; ++i) SPTS_TRY(mark(i));
  GemmArgs g1{b.xn, Nc, D, W->w_gate, W->w_up, L->F, SPTS_EPI_SWIGLU, b.act, nullptr, nullptr, 0.0, st};
  SPTS_TRY(launch_gemm(g1, s));
  SPTS_TRY(mark(14));
  GemmArgs g2{b.act, Nc, L->F, W->w_down, nullptr, D, SPTS_EPI_SCATTER_ADD, h, b.idx_a, nullptr, 0.0, st};
  SPTS_TRY(launch_gemm(g2, s));
  return mark(15);
}

}  // namespace

extern "C" {

size_t spts_layer_forward_workspace(const spts_layer_desc *L, int64_t Nc) {
  if (L == nullptr || Nc <= 0) return kStatusBytes;
  Carver cv(nullptr, 0);
  LayerBufs b;
  carve(cv, L, Nc, b);
  return cv.off;
}

spts_status spts_layer_forward(const spts_layer_desc *L, const spts_layer_weights *W, float *h, const int32_t *pos,
                               int64_t Nc, const spts_layer_outputs *out, void *ws, size_t ws_bytes,
                               spts_stream stream) {
  SPTS_TRY(check_layer(L, W, Nc));
  SPTS_REQUIRE(h && pos && aligned(h, 16) && aligned(pos, 4), SPTS_ERR_INVALID, "spts_layer_forward: bad h/pos");
  SPTS_TRY(check_ws(ws, ws_bytes, spts_layer_forward_workspace(L, Nc), "spts_layer_forward"));
  spts_layer_outputs none;
  memset(&none, 0, sizeof(none));
  const spts_layer_outputs &o = out ? *out : none;
  Carver cv(ws, ws_bytes);
  LayerBufs b;
  carve(cv, L, Nc, b);
  uint32_t *st = cv.status();
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (L->k == Nc && !o.s && !o.c && !o.f && !o.idx_attn && !o.idx_ffn && !o.k && !o.q_probe && L->n_salient == 0)
    return dense_layer(L, W, h, pos, Nc, o, b, st, s);
  const int D = L->D, P = L->P, hq = L->Hq * L->d, hk = L->Hkv * L->d;
  const int64_t k = L->k;
  float *sc = o.s ? o.s : b.s;
  int32_t *idx_a = o.idx_attn ? o.idx_attn : b.idx_a;
  void *osel = o.o_sel ? o.o_sel : b.osel;
  const float scale = 1.0f / sqrtf(static_cast<float>(L->d));
  auto mark = [&](int i) -> spts_status {
    if (o.stage_events != nullptr && o.stage_events[i] != nullptr)
      SPTS_CUDA_TRY(cudaEventRecord(static_cast<cudaEvent_t>(o.stage_events[i]), s));
    return SPTS_OK;
  };

  // Events 1..7 time stages that overlap the side stream's projections: when
  // any of them is requested every kernel runs on the caller's stream, so
  // the stage times add up.  Event 0 and events 8.. leave the side stream on.
  bool serial = false;
  if (o.stage_events != nullptr)
    for (int i = 1; i <= 7; ++i) serial = serial || o.stage_events[i] != nullptr;
  SideStream *side = nullptr;
  if (!serial) SPTS_TRY(side_stream(&side));
  // On any early return after the fork, still order the caller's stream
  // behind the side stream's work on the workspace.
  struct JoinGuard {
    SideStream *side;
    cudaStream_t s;
    bool joined;
    ~JoinGuard() {
      if (side && !joined) cudaStreamWaitEvent(s, side->v_done, 0);
    }
  } guard{side, s, false};

  // a1-a2: norm, K (+RoPE) / V for every candidate, Q (+RoPE) for the probe rows
  SPTS_TRY(mark(0));
  SPTS_TRY(launch_rmsnorm_rows(h, nullptr, Nc, D, W->norm_attn, L->eps, b.xn, s));
  SPTS_TRY(mark(1));
  const void *xtail = static_cast<const char *>(b.xn) + static_cast<size_t>(Nc - P) * D * 2;
  GemmArgs gq{xtail, P, D, W->w_q, nullptr, hq, SPTS_EPI_ROPE, b.qprobe, nullptr, pos + (Nc - P), L->theta, st};
  GemmArgs gv{b.xn, Nc, D, W->w_v, nullptr, hk, SPTS_EPI_STORE, b.vv, nullptr, nullptr, 0.0, st};
  const bool kv_active = L->kv_active_only != 0;  // V only for the active rows, later
  if (side) {  // fork: probe-Q and V projections on the side stream
    SPTS_CUDA_TRY(cudaEventRecord(side->fork, s));
    SPTS_CUDA_TRY(cudaStreamWaitEvent(side->s, side->fork, 0));
    SPTS_TRY(launch_gemm(gq, side->s));
    SPTS_CUDA_TRY(cudaEventRecord(side->qprobe_done, side->s));
    if (!kv_active) SPTS_TRY(launch_gemm(gv, side->s));
    SPTS_CUDA_TRY(cudaEventRecord(side->v_done, side->s));
  }
  GemmArgs gk{b.xn, Nc, D, W->w_k, nullptr, hk, SPTS_EPI_ROPE, b.kk, nullptr, pos, L->theta, st};
  SPTS_TRY(launch_gemm(gk, s));
  SPTS_TRY(mark(2));
  if (!side && !kv_active) SPTS_TRY(launch_gemm(gv, s));
  SPTS_TRY(mark(3));
  if (side) SPTS_CUDA_TRY(cudaStreamWaitEvent(s, side->qprobe_done, 0));
  else SPTS_TRY(launch_gemm(gq, s));
  if (L->n_salient > 0)
    SPTS_TRY(launch_inject_salience(b.kk, Nc, b.qprobe, P, L->Hq, L->Hkv, L->d, L->salient_rows, L->n_salient,
                                    L->salient_shift, st, s));
  if (o.k) SPTS_CUDA_TRY(cudaMemcpyAsync(o.k, b.kk, static_cast<size_t>(Nc) * hk * 2, cudaMemcpyDeviceToDevice, s));
  if (o.q_probe)
    SPTS_CUDA_TRY(cudaMemcpyAsync(o.q_probe, b.qprobe, static_cast<size_t>(P) * hq * 2, cudaMemcpyDeviceToDevice, s));
  SPTS_TRY(mark(4));

  // a3-a4: probe scores, MHA selection
  SPTS_TRY(launch_probe_bf16(b.qprobe, pos + (Nc - P), P, b.kk, pos, Nc, L->Hq, L->Hkv, scale, b.group, b.stats, st,
                             s));
  SPTS_TRY(launch_sum_groups(b.group, L->Hkv, Nc, sc, s));
  SPTS_TRY(mark(5));
  SPTS_TRY(launch_select_topk(sc, nullptr, SPTS_FUSE_NONE, 0.f, 0.f, Nc, k, P, idx_a, nullptr, nullptr, st, b.topk,
                              s));
  SPTS_TRY(mark(6));

  // a5-a7: Q for the selected rows, reduced attention, O projection into h
  SPTS_TRY(launch_gather_i32(pos, idx_a, k, b.qpos, s));
  SPTS_TRY(launch_gather_rows(b.xn, Nc, idx_a, k, static_cast<int64_t>(D) * 2, b.xsel, nullptr, nullptr, st, s));
  SPTS_TRY(mark(7));
  GemmArgs gqs{b.xsel, k, D, W->w_q, nullptr, hq, SPTS_EPI_ROPE, b.qsel, nullptr, b.qpos, L->theta, st};
  SPTS_TRY(launch_gemm(gqs, s));
  if (side) {  // join: V is ready
    SPTS_CUDA_TRY(cudaStreamWaitEvent(s, side->v_done, 0));
    guard.joined = true;
  }
  SPTS_TRY(mark(8));
  if (kv_active) {
    // keys and values of the active rows only: K gathered, V projected from
    // the gathered normalised rows, key positions = the active positions
    SPTS_TRY(launch_gather_rows(b.kk, Nc, idx_a, k, static_cast<int64_t>(hk) * 2, b.ksel, nullptr, nullptr, st, s));
    GemmArgs gvs{b.xsel, k, D, W->w_v, nullptr, hk, SPTS_EPI_STORE, b.vv, nullptr, nullptr, 0.0, st};
    SPTS_TRY(launch_gemm(gvs, s));
    SPTS_TRY(launch_attention_bf16(b.qsel, b.qpos, k, b.ksel, b.vv, b.qpos, k, L->Hq, L->Hkv, scale, osel, st, s));
  } else {
    SPTS_TRY(launch_attention_bf16(b.qsel, b.qpos, k, b.kk, b.vv, pos, Nc, L->Hq, L->Hkv, scale, osel, st, s));
  }
  SPTS_TRY(mark(9));
  GemmArgs go{osel, k, hq, W->w_o, nullptr, D, SPTS_EPI_SCATTER_ADD, h, idx_a, nullptr, 0.0, st};
  SPTS_TRY(launch_gemm(go, s));
  if (o.h_attn) SPTS_CUDA_TRY(cudaMemcpyAsync(o.h_attn, h, static_cast<size_t>(Nc) * D * 4, cudaMemcpyDeviceToDevice, s));
  SPTS_TRY(mark(10));
  if (L->F <= 0) {
    for (int i = 11; i < SPTS_LAYER_STAGE_EVENTS; ++i) SPTS_TRY(mark(i));
    return SPTS_OK;
  }

  // a8-a10: LTP score, fused FFN selection, reduced FFN
  float *c = o.c ? o.c : b.c;
  float *f = o.f ? o.f : b.f;
  int32_t *idx_f = o.idx_ffn ? o.idx_ffn : b.idx_f;
  // xn is free again: RMSNorm(h') under the FFN norm goes there.  When both
  // norms share one weight vector (or have none), RMSNorm(h') differs from
  // the attention input only on the k attention rows: renormalise just those.
  if (W->norm_ffn == W->norm_attn)
    SPTS_TRY(launch_rmsnorm_rows(h, idx_a, k, D, W->norm_ffn, L->eps, b.xn, s, /*scatter=*/true));
  else
    SPTS_TRY(launch_rmsnorm_rows(h, nullptr, Nc, D, W->norm_ffn, L->eps, b.xn, s));
  SPTS_TRY(mark(11));
  SPTS_TRY(launch_ltp_bf16(b.xn, Nc, D, W->ltp_a, L->r, W->ltp_b, L->ltp_dout > 0 ? L->ltp_dout : D, c, st, s,
                           L->ltp_top_m, b.gram));
  SPTS_TRY(mark(12));
  if (L->fuse == SPTS_FUSE_SEQUENTIAL) {
    const int64_t pool = L->seq_pool > 0 ? L->seq_pool : std::min<int64_t>(Nc, 2 * k);
    SPTS_TRY(launch_select_sequential(sc, c, Nc, pool, k, P, idx_f, b.topk, st, s));
    SPTS_CUDA_TRY(cudaMemcpyAsync(f, c, static_cast<size_t>(Nc) * 4, cudaMemcpyDeviceToDevice, s));
  } else {
    SPTS_TRY(launch_select_topk(sc, c, L->fuse, L->w_a, L->w_b, Nc, k, P, idx_f, f, nullptr, st, b.topk, s));
  }
  SPTS_TRY(launch_gather_rows(b.xn, Nc, idx_f, k, static_cast<int64_t>(D) * 2, b.xsel, nullptr, nullptr, st, s));
  SPTS_TRY(mark(13));
  GemmArgs g1{b.xsel, k, D, W->w_gate, W->w_up, L->F, SPTS_EPI_SWIGLU, b.act, nullptr, nullptr, 0.0, st};
  SPTS_TRY(launch_gemm(g1, s));
  SPTS_TRY(mark(14));
  GemmArgs g2{b.act, k, L->F, W->w_down, nullptr, D, SPTS_EPI_SCATTER_ADD, h, idx_f, nullptr, 0.0, st};
  SPTS_TRY(launch_gemm(g2, s));
  return mark(15);
}

// ---------------------------------------------------------------- bf16 residual boundary
// The layer on a bf16 residual stream at the boundary: h is converted to an
// fp32 copy in the workspace, spts_layer_forward runs on the copy, and the
// rows the layer changed (its attention rows and FFN rows; every row at
// k == Nc) are rounded back to bf16 in place.  Rows it skipped are not
// touched, so they keep their bf16 input exactly.
size_t spts_layer_forward_bf16io_workspace(const spts_layer_desc *L, int64_t Nc) {
  if (L == nullptr || Nc <= 0) return kStatusBytes;
  return Carver::round(spts_layer_forward_workspace(L, Nc)) + Carver::round(static_cast<size_t>(Nc) * L->D * 4) +
         2 * Carver::round(static_cast<size_t>(L->k > 0 ? L->k : 1) * 4);
}

spts_status spts_layer_forward_bf16io(const spts_layer_desc *L, const spts_layer_weights *W, void *h,
                                      const int32_t *pos, int64_t Nc, const spts_layer_outputs *out, void *ws,
                                      size_t ws_bytes, spts_stream stream) {
  const char *who = "spts_layer_forward_bf16io";
  SPTS_TRY(check_layer(L, W, Nc));
  SPTS_REQUIRE(h && pos && aligned(h, 16) && aligned(pos, 4), SPTS_ERR_INVALID, "%s: bad h/pos", who);
  SPTS_TRY(check_ws(ws, ws_bytes, spts_layer_forward_bf16io_workspace(L, Nc), who));
  const size_t lw = Carver::round(spts_layer_forward_workspace(L, Nc));
  char *extra = static_cast<char *>(ws) + lw;
  float *hf = reinterpret_cast<float *>(extra);
  extra += Carver::round(static_cast<size_t>(Nc) * L->D * 4);
  int32_t *ia = reinterpret_cast<int32_t *>(extra);
  int32_t *iff = reinterpret_cast<int32_t *>(extra + Carver::round(static_cast<size_t>(L->k > 0 ? L->k : 1) * 4));
  uint32_t *st = static_cast<uint32_t *>(ws);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  SPTS_TRY(launch_bf16_to_f32(h, Nc * L->D, hf, s));
  spts_layer_outputs o;
  if (out) o = *out;
  else memset(&o, 0, sizeof(o));
  const bool all_rows = L->k == Nc;  // keep 1.0: every row changes (and the dense path stays available)
  if (!all_rows) {
    if (!o.idx_attn) o.idx_attn = ia;
    if (L->F > 0 && !o.idx_ffn) o.idx_ffn = iff;
  }
  SPTS_TRY(spts_layer_forward(L, W, hf, pos, Nc, &o, ws, lw, stream));
  if (all_rows) {
    SPTS_TRY(launch_iota_i32(ia, Nc, s));  // k == Nc: ia holds Nc entries
    return launch_rows_f32_to_bf16(hf, ia, Nc, Nc, L->D, h, st, s);
  }
  SPTS_TRY(launch_rows_f32_to_bf16(hf, o.idx_attn, L->k, Nc, L->D, h, st, s));
  if (L->F > 0) SPTS_TRY(launch_rows_f32_to_bf16(hf, o.idx_ffn, L->k, Nc, L->D, h, st, s));
  return SPTS_OK;
}

// ---------------------------------------------------------------- MSDP
size_t spts_msdp_forward_workspace(const spts_layer_desc *L, int64_t N) {
  if (L == nullptr || N <= 0) return kStatusBytes;
  spts_layer_desc l = *L;
  l.k = N;  // the largest k any stage can use
  const size_t lw = Carver::round(spts_layer_forward_workspace(&l, N));
  return lw + Carver::round(static_cast<size_t>(N) * L->D * 4) + 3 * Carver::round(static_cast<size_t>(N) * 4);
}

spts_status spts_msdp_forward(const spts_layer_desc *L, const spts_layer_weights *W, int n_layers,
                              int layers_per_stage, const int64_t *stage_k, int n_stages, float *h, int32_t *pos,
                              int64_t N, int32_t *stage_pos, void *ws, size_t ws_bytes, spts_stream stream) {
  const char *who = "spts_msdp_forward";
  SPTS_REQUIRE(L && W && stage_k && h && pos, SPTS_ERR_INVALID, "%s: NULL argument", who);
  SPTS_REQUIRE(n_stages >= 1 && layers_per_stage >= 1 && n_layers == n_stages * layers_per_stage, SPTS_ERR_SHAPE,
               "%s: need n_layers == n_stages * layers_per_stage", who);
  int64_t prev = N;
  for (int s = 0; s < n_stages; ++s) {
    SPTS_REQUIRE(stage_k[s] >= L->P && stage_k[s] <= prev, SPTS_ERR_SHAPE,
                 "%s: stage %d keeps %lld rows of %lld (need P <= k_s <= |C_s|)", who, s,
                 static_cast<long long>(stage_k[s]), static_cast<long long>(prev));
    prev = stage_k[s];
  }
  SPTS_REQUIRE(L->F > 0, SPTS_ERR_SHAPE, "%s: pruning uses the fused FFN score, so F must be > 0", who);
  SPTS_TRY(check_ws(ws, ws_bytes, spts_msdp_forward_workspace(L, N), who));
  spts_layer_desc lmax = *L;
  lmax.k = N;
  const size_t lw = Carver::round(spts_layer_forward_workspace(&lmax, N));
  char *extra = static_cast<char *>(ws) + lw;
  float *h2 = reinterpret_cast<float *>(extra);
  extra += Carver::round(static_cast<size_t>(N) * L->D * 4);
  int32_t *pos2 = reinterpret_cast<int32_t *>(extra);
  extra += Carver::round(static_cast<size_t>(N) * 4);
  float *f = reinterpret_cast<float *>(extra);
  extra += Carver::round(static_cast<size_t>(N) * 4);
  int32_t *kept = reinterpret_cast<int32_t *>(extra);
  uint32_t *st = static_cast<uint32_t *>(ws);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);

  float *ha = h, *hb = h2;
  int32_t *pa = pos, *pb = pos2;
  int64_t Nc = N, out_off = 0;
  int li = 0;
  for (int stg = 0; stg < n_stages; ++stg) {
    spts_layer_desc d = *L;
    d.k = stage_k[stg];
    d.n_salient = 0;
    d.salient_rows = nullptr;
    spts_layer_outputs o;
    memset(&o, 0, sizeof(o));
    o.f = f;
    for (int l = 0; l < layers_per_stage; ++l, ++li) SPTS_TRY(spts_layer_forward(&d, &W[li], ha, pa, Nc, &o, ws, lw, stream));
    // stage boundary: C_{s+1} = top-k_s of C_s by the last layer's fused score
    // the layers are done with their workspace: its top-k scratch serves the prune
    Carver lcv(ws, lw);
    LayerBufs lb;
    carve(lcv, &lmax, N, lb);
    SPTS_TRY(launch_select_topk(f, nullptr, SPTS_FUSE_NONE, 0.f, 0.f, Nc, d.k, L->P, kept, nullptr, nullptr, st,
                                lb.topk, s));
    SPTS_TRY(launch_gather_rows(ha, Nc, kept, d.k, static_cast<int64_t>(L->D) * 4, hb, pa, pb, st, s));
    if (stage_pos)
      SPTS_CUDA_TRY(cudaMemcpyAsync(stage_pos + out_off, pb, static_cast<size_t>(d.k) * 4, cudaMemcpyDeviceToDevice, s));
    out_off += d.k;
    std::swap(ha, hb);
    std::swap(pa, pb);
    Nc = d.k;
  }
  if (ha != h) {
    SPTS_CUDA_TRY(cudaMemcpyAsync(h, ha, static_cast<size_t>(Nc) * L->D * 4, cudaMemcpyDeviceToDevice, s));
    SPTS_CUDA_TRY(cudaMemcpyAsync(pos, pa, static_cast<size_t>(Nc) * 4, cudaMemcpyDeviceToDevice, s));
  }
  return SPTS_OK;
}

// ---------------------------------------------------------------- layer schedule
size_t spts_schedule_forward_workspace(const spts_layer_desc *L, int64_t N) {
  if (L == nullptr || N <= 0) return kStatusBytes;
  spts_layer_desc l = *L;
  l.k = N;
  const size_t lw = Carver::round(spts_layer_forward_workspace(&l, N));
  return lw + Carver::round(static_cast<size_t>(N) * L->D * 4) + 4 * Carver::round(static_cast<size_t>(N) * 4);
}

spts_status spts_schedule_forward(const spts_layer_desc *L, const spts_layer_weights *W, int n_layers, int first_skip,
                                  const int *stage_ends, const int64_t *budgets, int n_stages, int64_t after_last,
                                  float *h, int32_t *pos, int64_t N, int64_t *n_out, int32_t *sel_pos,
                                  int64_t sel_cap, int64_t *sel_len, void *ws, size_t ws_bytes, spts_stream stream) {
  const char *who = "spts_schedule_forward";
  SPTS_REQUIRE(L && W && stage_ends && budgets && h && pos && n_out, SPTS_ERR_INVALID, "%s: NULL argument", who);
  SPTS_REQUIRE(n_stages >= 1 && n_layers >= 1 && first_skip >= 0 && first_skip <= stage_ends[0] &&
                   stage_ends[n_stages - 1] < n_layers,
               SPTS_ERR_SHAPE, "%s: need first_skip <= stage_ends[0] and stage_ends[last] < n_layers", who);
  for (int st = 0; st < n_stages; ++st) {
    SPTS_REQUIRE(st == 0 || stage_ends[st] > stage_ends[st - 1], SPTS_ERR_SHAPE, "%s: stage ends must ascend", who);
    SPTS_REQUIRE(budgets[st] >= L->P, SPTS_ERR_SHAPE, "%s: every budget must be >= P", who);
  }
  SPTS_REQUIRE(after_last >= L->P, SPTS_ERR_SHAPE, "%s: after_last must be >= P", who);
  SPTS_REQUIRE(L->F > 0, SPTS_ERR_SHAPE, "%s: pruning uses the fused FFN score, so F must be > 0", who);
  SPTS_REQUIRE(sel_pos == nullptr || sel_len != nullptr, SPTS_ERR_INVALID, "%s: sel_pos needs sel_len", who);
  SPTS_TRY(check_ws(ws, ws_bytes, spts_schedule_forward_workspace(L, N), who));
  spts_layer_desc lmax = *L;
  lmax.k = N;
  const size_t lw = Carver::round(spts_layer_forward_workspace(&lmax, N));
  char *extra = static_cast<char *>(ws) + lw;
  float *h2 = reinterpret_cast<float *>(extra);
  extra += Carver::round(static_cast<size_t>(N) * L->D * 4);
  int32_t *pos2 = reinterpret_cast<int32_t *>(extra);
  extra += Carver::round(static_cast<size_t>(N) * 4);
  float *f = reinterpret_cast<float *>(extra);
  extra += Carver::round(static_cast<size_t>(N) * 4);
  int32_t *kept = reinterpret_cast<int32_t *>(extra);
  extra += Carver::round(static_cast<size_t>(N) * 4);
  int32_t *idx_a = reinterpret_cast<int32_t *>(extra);
  uint32_t *st = static_cast<uint32_t *>(ws);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);

  float *ha = h, *hb = h2;
  int32_t *pa = pos, *pb = pos2;
  int64_t Nc = N, sel_off = 0;
  int stage = 0;
  for (int l = 0; l < n_layers; ++l) {
    const bool skip = l >= first_skip && stage < n_stages && l <= stage_ends[stage];
    spts_layer_desc d = *L;
    d.n_salient = 0;
    d.salient_rows = nullptr;
    spts_layer_outputs o;
    memset(&o, 0, sizeof(o));
    if (sel_len) sel_len[l] = 0;
    if (!skip) {  // a full layer over the current tokens (the dense path)
      d.k = Nc;
      SPTS_TRY(spts_layer_forward(&d, &W[l], ha, pa, Nc, &o, ws, lw, stream));
      continue;
    }
    d.k = std::min<int64_t>(budgets[stage], Nc);
    const bool stage_end = l == stage_ends[stage];
    o.idx_attn = idx_a;
    if (stage_end) o.f = f;
    SPTS_TRY(spts_layer_forward(&d, &W[l], ha, pa, Nc, &o, ws, lw, stream));
    if (sel_pos) {  // positions of this layer's attention set (consecutive-layer overlap diagnostics)
      SPTS_REQUIRE(sel_off + d.k <= sel_cap, SPTS_ERR_SHAPE, "%s: sel_pos holds %lld positions, needs more", who,
                   static_cast<long long>(sel_cap));
      SPTS_TRY(launch_gather_i32(pa, idx_a, d.k, sel_pos + sel_off, s));
      sel_len[l] = d.k;
      sel_off += d.k;
    }
    if (stage_end) {  // prune: the next stage's candidates (after the last: the tokens kept)
      const int64_t k_next = std::min<int64_t>(stage + 1 < n_stages ? budgets[stage] : after_last, Nc);
      Carver lcv(ws, lw);  // the layers are done with their workspace: its top-k scratch serves the prune
      LayerBufs lb;
      carve(lcv, &lmax, N, lb);
      SPTS_TRY(launch_select_topk(f, nullptr, SPTS_FUSE_NONE, 0.f, 0.f, Nc, k_next, L->P, kept, nullptr, nullptr, st,
                                  lb.topk, s));
      SPTS_TRY(launch_gather_rows(ha, Nc, kept, k_next, static_cast<int64_t>(L->D) * 4, hb, pa, pb, st, s));
      std::swap(ha, hb);
      std::swap(pa, pb);
      Nc = k_next;
      ++stage;
    }
  }
  if (ha != h) {
    SPTS_CUDA_TRY(cudaMemcpyAsync(h, ha, static_cast<size_t>(Nc) * L->D * 4, cudaMemcpyDeviceToDevice, s));
    SPTS_CUDA_TRY(cudaMemcpyAsync(pos, pa, static_cast<size_t>(Nc) * 4, cudaMemcpyDeviceToDevice, s));
  }
  *n_out = Nc;
  return SPTS_OK;
}

}  // extern "C"
