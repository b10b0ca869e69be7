"""CPU checks of the C ABI: the library loads, exports every entry point that
include/tq.h declares, sizes workspaces and rejects bad arguments before any
device work (no GPU needed for these paths)."""
import ctypes as C
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "tq.h")).read()
    return re.findall(r"^TQ_API\s+[\w\s\*]+?\b(tq_\w+)\s*\(", src, flags=re.M)


def test_header_declares_the_boundary():
    names = set(_declared())
    for must in ("tq_build_codebook", "tq_encode", "tq_score", "tq_topk", "tq_decode",
                 "tq_workspace_bytes", "tq_status_str"):
        assert must in names


def test_library_exports_every_declared_symbol(tq_lib):
    lib = C.CDLL(tq_lib.binding.LIB_PATH)
    for name in _declared():
        assert hasattr(lib, name), name
    assert set(_declared()) == set(tq_lib.binding.EXPORTS)


def test_status_strings(tq_lib):
    B = tq_lib.binding
    for s in (B.TQ_OK, B.TQ_ERR_ARG, B.TQ_ERR_UNSUPPORTED, B.TQ_ERR_WORKSPACE, B.TQ_ERR_CUDA,
              B.TQ_ERR_DEVICE_TIMEOUT, B.TQ_ERR_MISMATCH):
        assert B.tq_status_str(s) and B.tq_status_str(s) != "unknown status"
    assert B.tq_status_str(12345) == "unknown status"


def test_codebook_struct_layout(tq_lib, tmp_path):
    """The binding's struct matches the header's, as a C compiler lays it out."""
    B = tq_lib.binding
    fields = [f for f, _ in B.tq_codebook_t._fields_]
    src = tmp_path / "layout.c"
    src.write_text(
        "#include <stdio.h>\n#include <stddef.h>\n#include \"tq.h\"\n"
        "int main(void) {\n  printf(\"%zu\\n\", sizeof(tq_codebook_t));\n"
        + "".join(f"  printf(\"%zu\\n\", offsetof(tq_codebook_t, {f}));\n" for f in fields)
        + "  return 0;\n}\n")
    exe = tmp_path / "layout"
    subprocess.check_call(["gcc", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)])
    got = [int(v) for v in subprocess.check_output([str(exe)]).split()]
    assert got[0] == C.sizeof(B.tq_codebook_t) == 304
    assert got[1:] == [getattr(B.tq_codebook_t, f).offset for f in fields]


def test_workspace_sizes(tq_lib):
    B = tq_lib.binding
    big = (1 << 64) - 1
    assert B.tq_workspace_bytes(B.TQ_OP_BUILD, 128, 4, 1, 0, 0, 0) >= 2 * 128 * 128 * 8
    assert B.tq_workspace_bytes(B.TQ_OP_ENCODE, 100, 4, 1, 10, 0, 0) == big
    assert B.tq_workspace_bytes(B.TQ_OP_ENCODE, 128, 5, 1, 10, 0, 0) == big
    e1 = B.tq_workspace_bytes(B.TQ_OP_ENCODE, 128, 4, 1, 1000, 0, 0)
    e2 = B.tq_workspace_bytes(B.TQ_OP_ENCODE, 128, 4, 1, 10 ** 7, 0, 0)
    assert 0 < e1 < e2 and e2 == B.tq_workspace_bytes(B.TQ_OP_ENCODE, 128, 4, 1, 10 ** 8, 0, 0)
    s = B.tq_workspace_bytes(B.TQ_OP_SCORE, 128, 4, 8, 32768, 4, 0)
    assert s >= 2 * 8 * 4 * 128 * 4
    t = B.tq_workspace_bytes(B.TQ_OP_TOPK, 128, 4, 1, 10 ** 6, 1024, 10)
    assert t >= 1024 * ((10 ** 6 + 1023) // 1024) * 10 * 12
    assert B.tq_workspace_bytes(99, 128, 4, 1, 1, 1, 1) == big
    # scores + top-k: the top-k workspace without room for the scores
    st = B.tq_workspace_bytes(B.TQ_OP_SCORE_TOPK, 128, 4, 8, 32768, 4, 10)
    tt = B.tq_workspace_bytes(B.TQ_OP_TOPK, 128, 4, 8, 32768, 4, 10)
    assert 0 < st and st + 8 * 4 * 32768 * 4 <= tt
    # decode attention: d = 128 only, n >= 1; holds the logits [G][nq][n]
    a = B.tq_workspace_bytes(B.TQ_OP_ATTENTION, 128, 4, 8, 131072, 4, 0)
    assert a >= 8 * 4 * 131072 * 4 + s
    assert B.tq_workspace_bytes(B.TQ_OP_ATTENTION, 256, 4, 1, 100, 4, 0) == big
    assert B.tq_workspace_bytes(B.TQ_OP_ATTENTION, 128, 4, 1, 0, 4, 0) == big


def test_bad_arguments_rejected_without_device_work(tq_lib):
    B = tq_lib.binding
    cb = B.tq_codebook_t()
    lib = B.lib
    # unsupported shapes: rejected before any CUDA call
    assert lib.tq_build_codebook(100, 4, 0, 1, C.byref(cb), 1, 1, 1, 1 << 30, None) == B.TQ_ERR_UNSUPPORTED
    assert lib.tq_build_codebook(128, 5, 0, 1, C.byref(cb), 1, 1, 1, 1 << 30, None) == B.TQ_ERR_UNSUPPORTED
    assert lib.tq_build_codebook(128, 4, 0, 0, C.byref(cb), 1, 1, 1, 1 << 30, None) == B.TQ_ERR_ARG
    assert lib.tq_build_codebook(128, 4, 0, 1, None, 1, 1, 1, 1 << 30, None) == B.TQ_ERR_ARG
    assert lib.tq_build_codebook(128, 4, 0, 1, C.byref(cb), 1, 1, 1, 16, None) == B.TQ_ERR_WORKSPACE
    # fractional widths: b - 1/2 with 2 <= b <= 4, inner-product quantizer only
    assert lib.tq_build_codebook_split(128, 1, 0, 1, C.byref(cb), 1, 1, 1, 1 << 30, None) == B.TQ_ERR_UNSUPPORTED
    assert lib.tq_build_codebook_split(96, 3, 0, 1, C.byref(cb), 1, 1, 1, 1 << 30, None) == B.TQ_ERR_UNSUPPORTED
    assert lib.tq_build_codebook_split(128, 3, 0, 1, C.byref(cb), 1, None, 1, 1 << 30, None) == B.TQ_ERR_ARG
    assert lib.tq_build_codebook_split(128, 3, 0, 1, C.byref(cb), 1, 1, 1, 16, None) == B.TQ_ERR_WORKSPACE
    scb = B.tq_codebook_t()
    scb.d, scb.b, scb.groups, scb.levels, scb.variant, scb.split = 128, 3, 1, 4, B.TQ_VARIANT_MSE, 1
    assert lib.tq_encode(C.byref(scb), 1, 1, 1, 10, 1, 0, 1, 1, 1, 1, 1 << 30, None) == B.TQ_ERR_UNSUPPORTED
    scb.variant, scb.b = B.TQ_VARIANT_PROD, 1
    assert lib.tq_encode(C.byref(scb), 1, 1, 1, 10, 1, 0, 1, 1, 1, 1, 1 << 30, None) == B.TQ_ERR_UNSUPPORTED
    # a codebook that was never built: d = 0
    assert lib.tq_encode(C.byref(cb), 1, 1, 1, 10, 1, 0, 1, 1, 1, 1, 1 << 30, None) == B.TQ_ERR_UNSUPPORTED
    cb.d, cb.b, cb.groups, cb.levels = 128, 4, 1, 8
    assert lib.tq_encode(C.byref(cb), 1, 1, 2, 10, 1, 0, 1, 1, 1, 1, 1 << 30, None) == B.TQ_ERR_MISMATCH
    assert lib.tq_encode(C.byref(cb), 1, 1, 1, 10, 1, 7, 1, 1, 1, 1, 1 << 30, None) == B.TQ_ERR_ARG
    assert lib.tq_encode(C.byref(cb), 1, 1, 1, -1, 1, 0, 1, 1, 1, 1, 1 << 30, None) == B.TQ_ERR_ARG
    assert lib.tq_encode(C.byref(cb), 1, 1, 1, 10, None, 0, 1, 1, 1, 1, 1 << 30, None) == B.TQ_ERR_ARG
    assert lib.tq_encode(C.byref(cb), 1, 1, 1, 10, 1, 0, 1, 1, 1, 1, 8, None) == B.TQ_ERR_WORKSPACE
    assert lib.tq_encode(C.byref(cb), 1, 1, 1, 0, None, 0, None, None, None, None, 0, None) == B.TQ_OK
    assert lib.tq_score(C.byref(cb), 1, 1, 1, 10, 1, 1, 1, 4, 1, 0, 1, 1, 8, None) == B.TQ_ERR_WORKSPACE
    assert lib.tq_score(C.byref(cb), 1, 1, 1, 10, 1, 1, 1, 0, 1, 0, 1, 1, 8, None) == B.TQ_OK
    assert lib.tq_topk(C.byref(cb), 1, 1, 1, 10, 1, 1, 1, 4, 1, 0, 0, 1, 1, 1, 1 << 30, None) == B.TQ_ERR_ARG
    assert lib.tq_topk(C.byref(cb), 1, 1, 1, 10, 1, 1, 1, 4, 1, 0, 11, 1, 1, 1, 1 << 30, None) == B.TQ_ERR_ARG
    assert lib.tq_topk(C.byref(cb), 1, 1, 1, 100, 1, 1, 1, 4, 1, 0, 33, 1, 1, 1, 1 << 30, None) == B.TQ_ERR_ARG
    assert lib.tq_decode(C.byref(cb), 1, 1, 1, 10, 1, 1, 1, 1, 1, 8, None) == B.TQ_ERR_WORKSPACE
    assert lib.tq_logits_fp32(96, 1, 10, 1, 1, 1, 0, 1, None) == B.TQ_ERR_UNSUPPORTED
    assert lib.tq_exact_topk(128, 1, 10, 1, 1, 1, 0, 20, 1, 1, 1, 1 << 30, None) == B.TQ_ERR_ARG
    # scores + top-k in one call: the score output is required
    assert lib.tq_score_topk(C.byref(cb), 1, 1, 1, 100, 1, 1, 1, 4, 1, 0, 10, None, 1, 1, 1,
                             1 << 30, None) == B.TQ_ERR_ARG
    assert lib.tq_score_topk(C.byref(cb), 1, 1, 1, 100, 1, 1, 1, 4, 1, 0, 33, 1, 1, 1, 1,
                             1 << 30, None) == B.TQ_ERR_ARG
    # merge of shard lists
    assert lib.tq_topk_merge(4, 2, 0, 1, 1, 1, 1, None) == B.TQ_ERR_ARG
    assert lib.tq_topk_merge(4, 2, 33, 1, 1, 1, 1, None) == B.TQ_ERR_ARG
    assert lib.tq_topk_merge(4, 0, 10, 1, 1, 1, 1, None) == B.TQ_ERR_ARG
    assert lib.tq_topk_merge(4, 2, 10, None, 1, 1, 1, None) == B.TQ_ERR_ARG
    assert lib.tq_topk_merge(0, 2, 10, None, None, None, None, None) == B.TQ_OK
    # decode attention: keys PROD, values MSE, d = 128, n >= 1, finite scale
    kcb, vcb = B.tq_codebook_t(), B.tq_codebook_t()
    kcb.d, kcb.b, kcb.groups, kcb.levels, kcb.variant = 128, 4, 1, 8, B.TQ_VARIANT_PROD
    vcb.d, vcb.b, vcb.groups, vcb.levels, vcb.variant = 128, 4, 1, 16, B.TQ_VARIANT_MSE

    def attn(k=kcb, v=vcb, G=1, n=10, nq=4, scale=0.1, ws=1 << 30):
        return lib.tq_attention_decode(C.byref(k), 1, 1, C.byref(v), 1, G, n, 1, 1, 1, 1, 1, nq,
                                       1, 0, scale, 1, 1, ws, None)
    assert attn(n=0) == B.TQ_ERR_ARG
    assert attn(nq=0) == B.TQ_ERR_ARG
    assert attn(k=vcb) == B.TQ_ERR_ARG
    assert attn(v=kcb) == B.TQ_ERR_ARG
    assert attn(G=2) == B.TQ_ERR_MISMATCH
    assert attn(scale=float("nan")) == B.TQ_ERR_ARG
    assert attn(ws=64) == B.TQ_ERR_WORKSPACE
    kcb.split = 1
    assert attn() == B.TQ_ERR_UNSUPPORTED
    kcb.split = 0
    kcb.d = 96
    assert attn() == B.TQ_ERR_UNSUPPORTED


def test_binding_raises_on_error(tq_lib):
    B = tq_lib.binding
    cb = B.tq_codebook_t()
    with pytest.raises(B.TQError) as e:
        B.tq_encode(cb, 1, 1, 1, 10, 1, 0, 1, 1, 1, 1, 1 << 30, None)
    assert e.value.status == B.TQ_ERR_UNSUPPORTED
