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
