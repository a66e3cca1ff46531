"""The C-ABI library loads without a GPU and exports every declared symbol."""

import ctypes
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "spts.h")
LIB = os.path.join(ROOT, "token_skipping_sparse_b200", "libspts.so")


def declared():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^SPTS_API[^;]*?\b(spts_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_six_calls():
    names = declared()
    for n in ("spts_probe_scores", "spts_ltp_scores", "spts_select_topk", "spts_reduced_attention",
              "spts_reduced_ffn", "spts_stage_prune"):
        assert n in names


def test_library_exports_every_declared_symbol():
    if not os.path.exists(LIB):
        import token_skipping_sparse_b200.build as b
        b.build()
    lib = ctypes.CDLL(LIB)
    missing = [n for n in declared() if not hasattr(lib, n)]
    assert not missing, f"not exported: {missing}"


def test_binding_loads_and_reports_version():
    import token_skipping_sparse_b200 as S
    assert S.version().count(".") == 2
    assert set(S._lib.EXPORTS) >= set(declared())


def test_host_validation_without_gpu():
    """Argument checks run on the host before any launch."""
    import token_skipping_sparse_b200 as S
    lib = S.lib
    r = lib.spts_select_topk(None, None, 0, 0.5, 0.5, 10, 3, 0, None, None, None, None, 0, None)
    assert r == S.ERR_INVALID and "NULL" in S.last_error()
    a = S.AttnDesc(S.BF16, 32, 8, 64, 0.0)
    r = lib.spts_reduced_attention(ctypes.byref(a), 16, 16, 1, 16, 16, 16, 1, 32, 256, 256, None)
    assert r == S.ERR_UNSUPPORTED
    r = lib.spts_linear(16, 4, 100, 16, None, 256, 0, 16, None, None, 0.0, None, 0, None)
    assert r == S.ERR_SHAPE


# Placeholder addresses: never dereferenced, each case fails an argument
# check on the host before any launch.  A16 is 16-byte aligned, M8 is not.
A16, B16, C16, D16, E16 = 0x100000, 0x200000, 0x300000, 0x400000, 0x500000
M8 = 0x600008


def _cases(S):
    lib = S.lib
    bf = S.AttnDesc(S.BF16, 32, 8, 128, 0.0)
    bad_g = S.AttnDesc(S.BF16, 30, 8, 128, 0.0)      # Hq % Hkv != 0
    bad_d = S.AttnDesc(S.F32, 32, 8, 96, 0.0)        # head dim not 64 / 128
    g16 = S.AttnDesc(S.BF16, 32, 2, 128, 0.0)        # 16 query heads per KV head
    ld = S.layer_desc(1024, 8, 2, 128, 1536, 64, 16, 300)
    lw = S.LayerWeights(*([A16] * 9 + [None, None]))
    ref = ctypes.byref
    return [
        # probe scores: descriptor, P range, alignment
        ("probe Hq % Hkv", lambda: lib.spts_probe_scores(ref(bad_g), A16, B16, 4, C16, D16, 100, E16, None, None, 0,
                                                          None), S.ERR_SHAPE, "Hq % Hkv"),
        ("probe head dim", lambda: lib.spts_probe_scores(ref(bad_d), A16, B16, 4, C16, D16, 100, E16, None, None, 0,
                                                          None), S.ERR_SHAPE, "head dim"),
        ("probe GQA ratio", lambda: lib.spts_probe_scores(ref(g16), A16, B16, 4, C16, D16, 100, E16, None, None, 0,
                                                           None), S.ERR_UNSUPPORTED, "Hq/Hkv"),
        ("probe P = 0", lambda: lib.spts_probe_scores(ref(bf), A16, B16, 0, C16, D16, 100, E16, None, None, 0, None),
         S.ERR_SHAPE, "P"),
        ("probe P > Nc", lambda: lib.spts_probe_scores(ref(bf), A16, B16, 8, C16, D16, 5, E16, None, None, 0, None),
         S.ERR_SHAPE, "P"),
        ("probe P > 128", lambda: lib.spts_probe_scores(ref(bf), A16, B16, 129, C16, D16, 500, E16, None, None, 0,
                                                         None), S.ERR_SHAPE, "P"),
        ("probe misaligned q", lambda: lib.spts_probe_scores(ref(bf), M8, B16, 4, C16, D16, 100, E16, None, None, 0,
                                                              None), S.ERR_INVALID, "misaligned"),
        ("probe NULL keys", lambda: lib.spts_probe_scores(ref(bf), A16, B16, 4, None, D16, 100, E16, None, None, 0,
                                                           None), S.ERR_INVALID, "NULL"),
        # LTP: dtype, rank, widths
        ("ltp fp32", lambda: lib.spts_ltp_scores(S.F32, A16, 10, 256, B16, 64, C16, 256, D16, None, 0, None),
         S.ERR_UNSUPPORTED, "bf16"),
        ("ltp rank 32", lambda: lib.spts_ltp_scores(S.BF16, A16, 10, 256, B16, 32, C16, 256, D16, None, 0, None),
         S.ERR_SHAPE, ""),
        ("ltp D % 64", lambda: lib.spts_ltp_scores(S.BF16, A16, 10, 200, B16, 64, C16, 256, D16, None, 0, None),
         S.ERR_SHAPE, ""),
        ("ltp NULL weights", lambda: lib.spts_ltp_scores(S.BF16, A16, 10, 256, None, 64, C16, 256, D16, None, 0,
                                                          None), S.ERR_INVALID, "NULL"),
        # selection: mode, sizes, weights
        ("topk mode", lambda: lib.spts_select_topk(A16, B16, 99, 0.5, 0.5, 10, 3, 0, C16, None, None, None, 0, None),
         S.ERR_INVALID, "fusion mode"),
        ("topk k > Nc", lambda: lib.spts_select_topk(A16, None, 0, 0.5, 0.5, 10, 11, 0, C16, None, None, None, 0,
                                                      None), S.ERR_SHAPE, "k <= Nc"),
        ("topk tail > k", lambda: lib.spts_select_topk(A16, None, 0, 0.5, 0.5, 10, 3, 4, C16, None, None, None, 0,
                                                        None), S.ERR_SHAPE, "force_tail"),
        ("topk fused needs s_b", lambda: lib.spts_select_topk(A16, None, 1, 0.5, 0.5, 10, 3, 0, C16, None, None,
                                                               None, 0, None), S.ERR_INVALID, "NULL"),
        ("topk inf weight", lambda: lib.spts_select_topk(A16, B16, 1, float("inf"), 0.5, 10, 3, 0, C16, None, None,
                                                          None, 0, None), S.ERR_INVALID, "non-finite"),
        ("sequential pool < k", lambda: lib.spts_select_sequential(A16, B16, 10, 2, 3, 0, C16, None, 0, None),
         S.ERR_SHAPE, ""),
        # reduced attention: aliasing, sizes
        ("attention o aliases q", lambda: lib.spts_reduced_attention(ref(bf), A16, B16, 4, C16, D16, E16, 10, A16,
                                                                      None, 0, None), S.ERR_INVALID, "alias"),
        ("attention k < 0", lambda: lib.spts_reduced_attention(ref(bf), A16, B16, -1, C16, D16, E16, 10, 0x700000,
                                                                None, 0, None), S.ERR_SHAPE, "bad sizes"),
        ("attention Nc = 0", lambda: lib.spts_reduced_attention(ref(bf), A16, B16, 1, C16, D16, E16, 0, 0x700000,
                                                                 None, 0, None), S.ERR_SHAPE, "bad sizes"),
        # reduced FFN: shapes, eps
        ("ffn D % 256", lambda: lib.spts_reduced_ffn(S.BF16, A16, 10, 128, B16, 3, None, 1e-5, C16, D16, E16, 256,
                                                      None, 0, None), S.ERR_SHAPE, "D % 256"),
        ("ffn k > Nc", lambda: lib.spts_reduced_ffn(S.BF16, A16, 10, 256, B16, 11, None, 1e-5, C16, D16, E16, 256,
                                                     None, 0, None), S.ERR_SHAPE, "k <= Nc"),
        ("ffn eps < 0", lambda: lib.spts_reduced_ffn(S.BF16, A16, 10, 256, B16, 3, None, -1.0, C16, D16, E16, 256,
                                                      None, 0, None), S.ERR_INVALID, "eps"),
        ("ffn fp32", lambda: lib.spts_reduced_ffn(S.F32, A16, 10, 256, B16, 3, None, 1e-5, C16, D16, E16, 256, None,
                                                   0, None), S.ERR_UNSUPPORTED, "bf16"),
        # stage prune: sizes, overlap of the output with the input rows
        ("prune k_keep > Nc", lambda: lib.spts_stage_prune(A16, 10, 11, 0, B16, C16, 16, D16, E16, None, None, 0,
                                                            None), S.ERR_SHAPE, "k_keep"),
        ("prune D % 4", lambda: lib.spts_stage_prune(A16, 10, 5, 0, B16, C16, 18, D16, E16, None, None, 0, None),
         S.ERR_SHAPE, "D % 4"),
        ("prune h_out overlaps h_in", lambda: lib.spts_stage_prune(A16, 10, 5, 0, B16, C16, 16, B16 + 64, E16, None,
                                                                    None, 0, None), S.ERR_INVALID, "overlaps"),
        # supporting calls
        ("rmsnorm D % 8", lambda: lib.spts_rmsnorm_rows(A16, None, 4, 12, None, 1e-5, B16, None), S.ERR_SHAPE,
         "D % 8"),
        ("rope odd d", lambda: lib.spts_rope(A16, 4, 2, 7, B16, 10000.0, None), S.ERR_SHAPE, "even d"),
        ("rope theta 0", lambda: lib.spts_rope(A16, 4, 2, 8, B16, 0.0, None), S.ERR_SHAPE, "theta"),
        ("gather row bytes", lambda: lib.spts_gather_rows(A16, 10, B16, 4, 24, C16, None, None), S.ERR_SHAPE,
         "multiple of 16"),
        ("linear K % 64", lambda: lib.spts_linear(A16, 16, 100, B16, None, 256, 0, C16, None, None, 0.0, None, 0,
                                                   None), S.ERR_SHAPE, "K % 64"),
        ("linear bad epilogue", lambda: lib.spts_linear(A16, 16, 64, B16, None, 256, 9, C16, None, None, 0.0, None, 0,
                                                         None), S.ERR_INVALID, "epilogue"),
        ("linear SwiGLU needs W_up", lambda: lib.spts_linear(A16, 16, 64, B16, None, 256, 2, C16, None, None, 0.0,
                                                              None, 0, None), S.ERR_INVALID, "W2"),
        ("linear RoPE needs positions", lambda: lib.spts_linear(A16, 16, 64, B16, None, 256, 1, C16, None, None,
                                                                 10000.0, None, 0, None), S.ERR_INVALID, "row_pos"),
        ("linear scatter needs rows", lambda: lib.spts_linear(A16, 16, 64, B16, None, 256, 3, C16, None, None, 0.0,
                                                               None, 0, None), S.ERR_INVALID, "rows"),
        ("linear N % 256", lambda: lib.spts_linear(A16, 16, 64, B16, None, 200, 0, C16, None, None, 0.0, None, 0,
                                                    None), S.ERR_SHAPE, "N % 256"),
        ("salience geometry", lambda: lib.spts_inject_salience(A16, 10, B16, 4, 32, 8, 96, None, 0, 1.0, None),
         S.ERR_SHAPE, "geometry"),
        # the layer on a bf16 residual: alignment of h, positions present
        ("bf16io misaligned h", lambda: lib.spts_layer_forward_bf16io(ref(ld), ref(lw), M8, A16, 1000, None, None, 0,
                                                                      None), S.ERR_INVALID, "bad h/pos"),
        ("bf16io NULL pos", lambda: lib.spts_layer_forward_bf16io(ref(ld), ref(lw), A16, None, 1000, None, None, 0,
                                                                  None), S.ERR_INVALID, "bad h/pos"),
        ("bf16io k > Nc", lambda: lib.spts_layer_forward_bf16io(ref(ld), ref(lw), A16, B16, 200, None, None, 0,
                                                                None), S.ERR_SHAPE, "P <= k <= Nc"),
    ]


def test_argument_checks_return_the_documented_codes():
    """Every entry point rejects bad arguments on the host with the status
    its header comment names, and sets a message naming the call."""
    import token_skipping_sparse_b200 as S
    for name, call, code, fragment in _cases(S):
        r = call()
        msg = S.last_error()
        assert r == code, (name, r, msg)
        assert msg.startswith("spts_"), (name, msg)
        assert fragment in msg, (name, msg)
