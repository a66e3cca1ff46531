"""ctypes binding of libspts.so -- argument marshalling only.

Every function here checks nothing the library does not check itself: it
turns torch tensors into raw device pointers, picks the current CUDA stream,
sizes the workspace with the library's own *_workspace() query, calls the C
entry point of the same name and raises SptsError on a non-zero status.  All
arithmetic runs in the library's CUDA kernels; there is no fallback path.
"""

from __future__ import annotations

import ctypes as C
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libspts.so")

OK, ERR_INVALID, ERR_SHAPE, ERR_UNSUPPORTED, ERR_CUDA, ERR_TIMEOUT, ERR_WORKSPACE = range(7)
F32, BF16 = 0, 1
FUSE_NONE, FUSE_MAXNORM_ADD, FUSE_MULTIPLY, FUSE_STD_ADD, FUSE_SEQUENTIAL = 0, 1, 2, 3, 4
EPI_STORE, EPI_ROPE, EPI_SWIGLU, EPI_SCATTER_ADD = 0, 1, 2, 3

EXPORTS = (
    "spts_version", "spts_last_error", "spts_check_device_status", "spts_debug_set_wait_limit_ns",
    "spts_debug_get_wait_limit_ns", "spts_launch_count",
    "spts_probe_scores", "spts_probe_scores_workspace", "spts_ltp_scores", "spts_ltp_scores_workspace",
    "spts_ltp_topm_scores", "spts_ltp_topm_scores_workspace",
    "spts_select_topk", "spts_select_topk_workspace", "spts_select_sequential", "spts_select_sequential_workspace",
    "spts_reduced_attention",
    "spts_reduced_attention_workspace", "spts_reduced_ffn", "spts_reduced_ffn_workspace", "spts_stage_prune",
    "spts_stage_prune_workspace", "spts_stage_prune_noalloc", "spts_rmsnorm_rows", "spts_rope", "spts_gather_rows", "spts_linear",
    "spts_linear_workspace", "spts_inject_salience", "spts_layer_forward", "spts_layer_forward_workspace",
    "spts_msdp_forward", "spts_msdp_forward_workspace", "spts_schedule_forward", "spts_schedule_forward_workspace",
    "spts_layer_forward_bf16io", "spts_layer_forward_bf16io_workspace", "spts_debug_exp2_poly",
)


class SptsError(RuntimeError):
    def __init__(self, status, message):
        super().__init__(f"spts status {status}: {message}")
        self.status = status


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with token_skipping_sparse_b200.build.build() "
                          "(there is no CPU fallback)")
    return C.CDLL(LIB_PATH)


lib = _load()

vp, sz, i64, i32, f32, f64, u64 = C.c_void_p, C.c_size_t, C.c_int64, C.c_int, C.c_float, C.c_double, C.c_uint64


class AttnDesc(C.Structure):
    _fields_ = [("dtype", C.c_int), ("Hq", C.c_int), ("Hkv", C.c_int), ("d", C.c_int), ("scale", C.c_float)]


class LayerDesc(C.Structure):
    _fields_ = [("D", C.c_int), ("Hq", C.c_int), ("Hkv", C.c_int), ("d", C.c_int), ("F", C.c_int),
                ("r", C.c_int), ("P", C.c_int), ("k", C.c_int64), ("fuse", C.c_int), ("w_a", C.c_float),
                ("w_b", C.c_float), ("eps", C.c_float), ("theta", C.c_double), ("salient_rows", C.c_void_p),
                ("n_salient", C.c_int64), ("salient_shift", C.c_float), ("ltp_dout", C.c_int),
                ("kv_active_only", C.c_int), ("ltp_top_m", C.c_int), ("seq_pool", C.c_int64)]


class LayerWeights(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in ("w_q", "w_k", "w_v", "w_o", "w_gate", "w_up", "w_down", "ltp_a",
                                          "ltp_b", "norm_attn", "norm_ffn")]


class LayerOutputs(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in ("s", "c", "f", "idx_attn", "idx_ffn", "o_sel", "h_attn", "k",
                                          "q_probe", "stage_events")]


LAYER_STAGE_EVENTS = 16
LAYER_STAGES = ("rmsnorm", "k_proj_rope", "v_proj", "probe_q_proj", "probe_scores", "select_mha", "gathers",
                "q_proj_rope", "reduced_attention", "o_proj_scatter", "rmsnorm_ffn", "ltp_scores",
                "select_ffn_gather", "gate_up_swiglu", "down_proj_scatter")


def _sig(name, res, args):
    fn = getattr(lib, name)
    fn.restype = res
    fn.argtypes = args
    return fn


AD = C.POINTER(AttnDesc)
_sig("spts_version", C.c_char_p, [])
_sig("spts_last_error", sz, [C.c_char_p, sz])
_sig("spts_check_device_status", i32, [vp, vp])
_sig("spts_debug_set_wait_limit_ns", None, [u64])
_sig("spts_debug_get_wait_limit_ns", u64, [])
_sig("spts_launch_count", u64, [])
_sig("spts_debug_exp2_poly", i32, [vp, i64, vp, vp])
_sig("spts_probe_scores", i32, [AD, vp, vp, i32, vp, vp, i64, vp, vp, vp, sz, vp])
_sig("spts_probe_scores_workspace", sz, [AD, i32, i64])
_sig("spts_ltp_scores", i32, [i32, vp, i64, i32, vp, i32, vp, i32, vp, vp, sz, vp])
_sig("spts_ltp_scores_workspace", sz, [i64, i32, i32, i32])
_sig("spts_ltp_topm_scores", i32, [i32, vp, i64, i32, vp, i32, vp, i32, i32, vp, vp, sz, vp])
_sig("spts_ltp_topm_scores_workspace", sz, [i64, i32, i32, i32])
_sig("spts_select_topk", i32, [vp, vp, i32, f32, f32, i64, i64, i64, vp, vp, vp, vp, sz, vp])
_sig("spts_select_topk_workspace", sz, [i64])
_sig("spts_select_sequential", i32, [vp, vp, i64, i64, i64, i64, vp, vp, sz, vp])
_sig("spts_select_sequential_workspace", sz, [i64])
_sig("spts_reduced_attention", i32, [AD, vp, vp, i64, vp, vp, vp, i64, vp, vp, sz, vp])
_sig("spts_reduced_attention_workspace", sz, [AD, i64, i64])
_sig("spts_reduced_ffn", i32, [i32, vp, i64, i32, vp, i64, vp, f32, vp, vp, vp, i32, vp, sz, vp])
_sig("spts_reduced_ffn_workspace", sz, [i64, i32, i32])
_sig("spts_stage_prune", i32, [vp, i64, i64, i64, vp, vp, i32, vp, vp, vp, vp, sz, vp])
_sig("spts_stage_prune_workspace", sz, [i64])
_sig("spts_stage_prune_noalloc", i32, [vp, i64, i64, i64, vp, vp, i32, vp, vp, vp, vp])
NOALLOC_MAX_NC = 262144
_sig("spts_rmsnorm_rows", i32, [vp, vp, i64, i32, vp, f32, vp, vp])
_sig("spts_rope", i32, [vp, i64, i32, i32, vp, f64, vp])
_sig("spts_gather_rows", i32, [vp, i64, vp, i64, i64, vp, vp, vp])
_sig("spts_linear", i32, [vp, i64, i32, vp, vp, i32, i32, vp, vp, vp, f64, vp, sz, vp])
_sig("spts_linear_workspace", sz, [])
_sig("spts_inject_salience", i32, [vp, i64, vp, i32, i32, i32, i32, vp, i64, f32, vp])
if hasattr(lib, "spts_layer_forward"):
    _sig("spts_layer_forward", i32, [C.POINTER(LayerDesc), C.POINTER(LayerWeights), vp, vp, i64,
                                     C.POINTER(LayerOutputs), vp, sz, vp])
    _sig("spts_layer_forward_workspace", sz, [C.POINTER(LayerDesc), i64])
    _sig("spts_msdp_forward", i32, [C.POINTER(LayerDesc), C.POINTER(LayerWeights), i32, i32, C.POINTER(C.c_int64),
                                    i32, vp, vp, i64, vp, vp, sz, vp])
    _sig("spts_msdp_forward_workspace", sz, [C.POINTER(LayerDesc), i64])
    _sig("spts_layer_forward_bf16io", i32, [C.POINTER(LayerDesc), C.POINTER(LayerWeights), vp, vp, i64,
                                            C.POINTER(LayerOutputs), vp, sz, vp])
    _sig("spts_layer_forward_bf16io_workspace", sz, [C.POINTER(LayerDesc), i64])
_sig("spts_schedule_forward", i32, [C.POINTER(LayerDesc), C.POINTER(LayerWeights), i32, i32, C.POINTER(C.c_int),
                                    C.POINTER(C.c_int64), i32, i64, vp, vp, i64, C.POINTER(C.c_int64), vp, i64,
                                    C.POINTER(C.c_int64), vp, sz, vp])
_sig("spts_schedule_forward_workspace", sz, [C.POINTER(LayerDesc), i64])


# ---------------------------------------------------------------- helpers
def version():
    return lib.spts_version().decode()


def last_error():
    buf = C.create_string_buffer(1024)
    lib.spts_last_error(buf, 1024)
    return buf.value.decode(errors="replace")


def check(status):
    if status != OK:
        raise SptsError(status, last_error())


def ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def stream_ptr(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return C.c_void_p(s.cuda_stream)


_ws_lock = threading.Lock()
_ws_cache = {}


def workspace(nbytes, device=None):
    """A zero-initialised, per-device cached workspace of at least nbytes.

    Calls that use the cached workspace must be ordered on one stream; pass
    your own workspace tensor (torch.zeros(n, dtype=uint8)) to overlap calls.
    """
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    with _ws_lock:
        t = _ws_cache.get(dev)
        if t is None or t.numel() < nbytes:
            t = torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=dev)
            _ws_cache[dev] = t
        return t


def launch_count():
    return int(lib.spts_launch_count())


def debug_exp2_poly(x):
    """The reduced-attention softmax's FMA-pipe exp2 applied to a device fp32 tensor."""
    y = torch.empty_like(x)
    check(lib.spts_debug_exp2_poly(ptr(x), x.numel(), ptr(y), stream_ptr()))
    return y


def set_wait_limit_ns(ns):
    lib.spts_debug_set_wait_limit_ns(int(ns))


def get_wait_limit_ns():
    return int(lib.spts_debug_get_wait_limit_ns())


def check_device_status(ws=None, stream=None):
    ws = workspace(256) if ws is None else ws
    check(lib.spts_check_device_status(ptr(ws), stream_ptr(stream)))


def _attn_desc(dtype, Hq, Hkv, d, scale):
    return AttnDesc(BF16 if dtype == torch.bfloat16 else F32, Hq, Hkv, d, 0.0 if scale is None else float(scale))


# ---------------------------------------------------------------- the six calls
def spts_probe_scores(q_probe, probe_pos, k, key_pos, scale=None, group_scores=False, ws=None):
    P, Hq, d = q_probe.shape
    Nc, Hkv, _ = k.shape
    a = _attn_desc(q_probe.dtype, Hq, Hkv, d, scale)
    s = torch.empty(Nc, dtype=torch.float32, device=k.device)
    g = torch.empty(Hkv, Nc, dtype=torch.float32, device=k.device) if group_scores else None
    n = lib.spts_probe_scores_workspace(C.byref(a), P, Nc)
    ws = workspace(n) if ws is None else ws
    check(lib.spts_probe_scores(C.byref(a), ptr(q_probe), ptr(probe_pos), P, ptr(k), ptr(key_pos), Nc, ptr(s),
                                ptr(g), ptr(ws), ws.numel(), stream_ptr()))
    return (s, g) if group_scores else s


def spts_ltp_scores(x, A, B, ws=None):
    Nc, D = x.shape
    r, Dout = A.shape[0], B.shape[0]
    c = torch.empty(Nc, dtype=torch.float32, device=x.device)
    n = lib.spts_ltp_scores_workspace(Nc, D, r, Dout)
    ws = workspace(n) if ws is None else ws
    check(lib.spts_ltp_scores(BF16, ptr(x), Nc, D, ptr(A), r, ptr(B), Dout, ptr(c), ptr(ws), ws.numel(),
                              stream_ptr()))
    return c


def spts_ltp_topm_scores(x, A, B, top_m, ws=None):
    """Sum of the top_m largest |y| per row of y = (x A^T) B^T (top-rho saliency)."""
    Nc, D = x.shape
    r, Dout = A.shape[0], B.shape[0]
    c = torch.empty(Nc, dtype=torch.float32, device=x.device)
    n = lib.spts_ltp_topm_scores_workspace(Nc, D, r, Dout)
    ws = workspace(n) if ws is None else ws
    check(lib.spts_ltp_topm_scores(BF16, ptr(x), Nc, D, ptr(A), r, ptr(B), Dout, int(top_m), ptr(c), ptr(ws),
                                   ws.numel(), stream_ptr()))
    return c


def spts_select_sequential(s_a, s_b, k_pool, k, force_tail, ws=None):
    """Top-k_pool by s_a (tail forced), then the top-k of that pool by s_b; indices ascending."""
    Nc = s_a.shape[0]
    idx = torch.empty(k, dtype=torch.int32, device=s_a.device)
    n = lib.spts_select_sequential_workspace(Nc)
    ws = workspace(n) if ws is None else ws
    check(lib.spts_select_sequential(ptr(s_a), ptr(s_b), Nc, k_pool, k, force_tail, ptr(idx), ptr(ws), ws.numel(),
                                     stream_ptr()))
    return idx


def spts_select_topk(s_a, k, force_tail, s_b=None, mode=FUSE_NONE, w_a=0.5, w_b=0.5, fused=False, kth=False,
                     ws=None):
    Nc = s_a.shape[0]
    idx = torch.empty(k, dtype=torch.int32, device=s_a.device)
    fo = torch.empty(Nc, dtype=torch.float32, device=s_a.device) if fused else None
    ko = torch.empty(1, dtype=torch.float32, device=s_a.device) if kth else None
    n = lib.spts_select_topk_workspace(Nc)
    ws = workspace(n) if ws is None else ws
    check(lib.spts_select_topk(ptr(s_a), ptr(s_b), mode, w_a, w_b, Nc, k, force_tail, ptr(idx), ptr(fo), ptr(ko),
                               ptr(ws), ws.numel(), stream_ptr()))
    out = [idx]
    if fused:
        out.append(fo)
    if kth:
        out.append(ko)
    return idx if len(out) == 1 else tuple(out)


def spts_reduced_attention(q_sel, q_pos, k, v, key_pos, scale=None, out=None, ws=None):
    m, Hq, d = q_sel.shape
    Nc, Hkv, _ = k.shape
    a = _attn_desc(q_sel.dtype, Hq, Hkv, d, scale)
    o = torch.empty_like(q_sel) if out is None else out
    n = lib.spts_reduced_attention_workspace(C.byref(a), m, Nc)
    ws = workspace(n) if ws is None else ws
    check(lib.spts_reduced_attention(C.byref(a), ptr(q_sel), ptr(q_pos), m, ptr(k), ptr(v), ptr(key_pos), Nc,
                                     ptr(o), ptr(ws), ws.numel(), stream_ptr()))
    return o


def spts_reduced_ffn(h, idx, norm_w, eps, w_gate, w_up, w_down, ws=None):
    Nc, D = h.shape
    F = w_gate.shape[0]
    k = idx.shape[0]
    n = lib.spts_reduced_ffn_workspace(k, D, F)
    ws = workspace(n) if ws is None else ws
    check(lib.spts_reduced_ffn(BF16, ptr(h), Nc, D, ptr(idx), k, ptr(norm_w), eps, ptr(w_gate), ptr(w_up),
                               ptr(w_down), F, ptr(ws), ws.numel(), stream_ptr()))
    return h


def spts_stage_prune(scores, k_keep, force_tail, h, pos, ws=None):
    Nc, D = h.shape
    h_out = torch.empty(k_keep, D, dtype=h.dtype, device=h.device)
    pos_out = torch.empty(k_keep, dtype=torch.int32, device=h.device)
    kept = torch.empty(k_keep, dtype=torch.int32, device=h.device)
    n = lib.spts_stage_prune_workspace(Nc)
    ws = workspace(n) if ws is None else ws
    check(lib.spts_stage_prune(ptr(scores), Nc, k_keep, force_tail, ptr(h), ptr(pos), D, ptr(h_out),
                               ptr(pos_out), ptr(kept), ptr(ws), ws.numel(), stream_ptr()))
    return h_out, pos_out, kept


def spts_stage_prune_noalloc(scores, k_keep, force_tail, h, pos, kept=None):
    """The allocation-free stage prune: no workspace; the kept indices go to
    the library's fixed device array unless `kept` (int32 [k_keep]) is given.
    Output tensors are allocated here by torch, as for every call of this
    binding; the C entry point itself allocates nothing."""
    Nc, D = h.shape
    h_out = torch.empty(k_keep, D, dtype=h.dtype, device=h.device)
    pos_out = torch.empty(k_keep, dtype=torch.int32, device=h.device)
    check(lib.spts_stage_prune_noalloc(ptr(scores), Nc, k_keep, force_tail, ptr(h), ptr(pos), D, ptr(h_out),
                                       ptr(pos_out), ptr(kept), stream_ptr()))
    return h_out, pos_out


# ---------------------------------------------------------------- supporting calls
def spts_rmsnorm_rows(x, w=None, eps=1e-5, rows=None):
    m = x.shape[0] if rows is None else rows.shape[0]
    D = x.shape[1]
    y = torch.empty(m, D, dtype=torch.bfloat16, device=x.device)
    check(lib.spts_rmsnorm_rows(ptr(x), ptr(rows), m, D, ptr(w), eps, ptr(y), stream_ptr()))
    return y


def spts_rope(x, pos, theta=500000.0):
    m, H, d = x.shape
    check(lib.spts_rope(ptr(x), m, H, d, ptr(pos), theta, stream_ptr()))
    return x


def spts_gather_rows(src, rows, ws=None):
    n_src = src.shape[0]
    m = rows.shape[0]
    row_bytes = src[0].numel() * src.element_size() if n_src else 16
    dst = torch.empty((m,) + tuple(src.shape[1:]), dtype=src.dtype, device=src.device)
    ws = workspace(256) if ws is None else ws
    check(lib.spts_gather_rows(ptr(src), n_src, ptr(rows), m, row_bytes, ptr(dst), ptr(ws), stream_ptr()))
    return dst


def spts_linear(A, W, epi=EPI_STORE, W2=None, out=None, rows=None, row_pos=None, theta=500000.0, ws=None):
    M, K = A.shape
    N = W.shape[0]
    if out is None:
        out = torch.empty(M, N, dtype=torch.bfloat16, device=A.device)
    ws = workspace(lib.spts_linear_workspace()) if ws is None else ws
    check(lib.spts_linear(ptr(A), M, K, ptr(W), ptr(W2), N, epi, ptr(out), ptr(rows), ptr(row_pos), theta,
                          ptr(ws), ws.numel(), stream_ptr()))
    return out


def spts_inject_salience(k, q_probe, rows, shift):
    Nc, Hkv, d = k.shape
    P, Hq, _ = q_probe.shape
    check(lib.spts_inject_salience(ptr(k), Nc, ptr(q_probe), P, Hq, Hkv, d, ptr(rows), rows.shape[0], shift,
                                   stream_ptr()))
    return k


# ---------------------------------------------------------------- the composed layer
def layer_desc(D, Hq, Hkv, d, F, r, P, k, fuse=FUSE_MAXNORM_ADD, w_a=0.5, w_b=0.5, eps=1e-5, theta=500000.0,
               salient_rows=None, salient_shift=0.0, ltp_dout=0, kv_active_only=False, ltp_top_m=0, seq_pool=0):
    n_sal = 0 if salient_rows is None else int(salient_rows.numel())
    desc = LayerDesc(D, Hq, Hkv, d, F, r, P, k, fuse, w_a, w_b, eps, theta,
                     None if n_sal == 0 else salient_rows.data_ptr(), n_sal, salient_shift, ltp_dout,
                     1 if kv_active_only else 0, int(ltp_top_m), int(seq_pool))
    desc._keep = salient_rows  # the descriptor holds a raw pointer: keep the tensor alive with it
    return desc


def layer_weights(w):
    """w: dict of device tensors named as the spts_layer_weights fields."""
    return LayerWeights(*[None if w.get(n) is None else w[n].data_ptr() for n, _ in LayerWeights._fields_])


def stage_events():
    """LAYER_STAGE_EVENTS timing events, created (recorded once) so their
    raw handles exist; pass them to spts_layer_forward(events=...)."""
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(LAYER_STAGE_EVENTS)]
    for e in evs:
        e.record()
    torch.cuda.synchronize()
    return evs


def spts_layer_forward(h, pos, desc, weights, outputs=False, ws=None, events=None):
    """Runs one layer in place on h [Nc, D] fp32; returns a dict of the
    optional outputs when outputs=True.  `events` (from stage_events(), or a
    list of LAYER_STAGE_EVENTS entries some of which are None) are recorded
    at the stage boundaries."""
    Nc = h.shape[0]
    out = None
    res = {}
    ev_arr = None
    if events is not None:
        ev_arr = (C.c_void_p * LAYER_STAGE_EVENTS)(*[e.cuda_event if e is not None else None for e in events])
    if outputs is not False or events is not None:
        out = LayerOutputs()
        out.stage_events = C.cast(ev_arr, C.c_void_p) if ev_arr is not None else None
    if isinstance(outputs, dict):          # caller-provided subset of the outputs
        res = outputs
        for n, t in res.items():
            setattr(out, n, t.data_ptr())
    elif outputs:
        dv = h.device
        k, hq = desc.k, desc.Hq * desc.d
        res = dict(s=torch.empty(Nc, dtype=torch.float32, device=dv),
                   c=torch.empty(Nc, dtype=torch.float32, device=dv),
                   f=torch.empty(Nc, dtype=torch.float32, device=dv),
                   idx_attn=torch.empty(k, dtype=torch.int32, device=dv),
                   idx_ffn=torch.empty(k, dtype=torch.int32, device=dv),
                   o_sel=torch.empty(k, desc.Hq, desc.d, dtype=torch.bfloat16, device=dv),
                   h_attn=torch.empty_like(h),
                   k=torch.empty(Nc, desc.Hkv, desc.d, dtype=torch.bfloat16, device=dv),
                   q_probe=torch.empty(desc.P, desc.Hq, desc.d, dtype=torch.bfloat16, device=dv))
        for n, t in res.items():
            setattr(out, n, t.data_ptr())
    w = weights if isinstance(weights, LayerWeights) else layer_weights(weights)
    n = lib.spts_layer_forward_workspace(C.byref(desc), Nc)
    ws = workspace(n) if ws is None else ws
    check(lib.spts_layer_forward(C.byref(desc), C.byref(w), ptr(h), ptr(pos), Nc,
                                 None if out is None else C.byref(out), ptr(ws), ws.numel(), stream_ptr()))
    return res


def spts_layer_forward_bf16io(h, pos, desc, weights, ws=None):
    """One layer in place on a bf16 residual h [Nc, D]: computed in fp32 on
    a workspace copy; the rows the layer changed are rounded back to bf16."""
    Nc = h.shape[0]
    w = weights if isinstance(weights, LayerWeights) else layer_weights(weights)
    n = lib.spts_layer_forward_bf16io_workspace(C.byref(desc), Nc)
    ws = workspace(n) if ws is None else ws
    check(lib.spts_layer_forward_bf16io(C.byref(desc), C.byref(w), ptr(h), ptr(pos), Nc, None, ptr(ws), ws.numel(),
                                        stream_ptr()))
    return h


def spts_msdp_forward(h, pos, desc, layer_weights_list, layers_per_stage, stage_k, stage_pos=False, ws=None):
    """MSDP over len(layer_weights_list) layers, in place on h [N, D] / pos [N].
    Returns (number of final candidates, per-stage candidate positions or None)."""
    N = h.shape[0]
    n_layers = len(layer_weights_list)
    ws_list = [w if isinstance(w, LayerWeights) else layer_weights(w) for w in layer_weights_list]
    W = (LayerWeights * n_layers)(*ws_list)
    ks = (C.c_int64 * len(stage_k))(*[int(k) for k in stage_k])
    sp = torch.empty(int(sum(stage_k)), dtype=torch.int32, device=h.device) if stage_pos else None
    n = lib.spts_msdp_forward_workspace(C.byref(desc), N)
    ws = workspace(n) if ws is None else ws
    check(lib.spts_msdp_forward(C.byref(desc), W, n_layers, layers_per_stage, ks, len(stage_k), ptr(h), ptr(pos),
                                N, ptr(sp), ptr(ws), ws.numel(), stream_ptr()))
    if sp is None:
        return int(stage_k[-1]), None
    out, off = [], 0
    for k in stage_k:
        out.append(sp[off:off + int(k)])
        off += int(k)
    return int(stage_k[-1]), out


def spts_schedule_forward(h, pos, desc, layer_weights_list, first_skip, stage_ends, budgets, after_last,
                          selections=False, ws=None):
    """A Table-B layer schedule over h [N, D] fp32 and pos [N] int32, in place.

    Returns the number of rows left (h[:n], pos[:n] hold them); with
    ``selections`` also the per-layer positions of every skipping layer's
    attention set (None for full layers)."""
    N = h.shape[0]
    n_layers = len(layer_weights_list)
    Ws = (LayerWeights * n_layers)(*[layer_weights(w) for w in layer_weights_list])
    ends = (C.c_int * len(stage_ends))(*stage_ends)
    buds = (C.c_int64 * len(budgets))(*budgets)
    n_out = C.c_int64(0)
    sel = sel_len = None
    cap = 0
    if selections:
        cap = sum(min(b, N) for b in budgets) * n_layers
        sel = torch.empty(cap, dtype=torch.int32, device=h.device)
        sel_len = (C.c_int64 * n_layers)()
    n = lib.spts_schedule_forward_workspace(C.byref(desc), N)
    ws = workspace(n) if ws is None else ws
    check(lib.spts_schedule_forward(C.byref(desc), Ws, n_layers, first_skip, ends, buds, len(stage_ends), after_last,
                                    ptr(h), ptr(pos), N, C.byref(n_out), ptr(sel) if sel is not None else None, cap,
                                    sel_len, ptr(ws), ws.numel(), stream_ptr()))
    if not selections:
        return int(n_out.value)
    out, off = [], 0
    for l in range(n_layers):
        m = int(sel_len[l])
        out.append(sel[off:off + m] if m else None)
        off += m
    return int(n_out.value), out
